// attn_bwd_noalloc: the backward for callers that cannot allocate device memory.
//
// attn_bwd needs a caller-provided workspace (status word, padded row terms,
// fp32 dQ accumulator). Some callers cannot obtain one: code that runs inside
// a host framework whose device memory is fully reserved by that framework's
// own pool and that is not allowed to call cudaMalloc (a plugin or custom
// operator), or latency-critical code that must not pay for an allocation
// (cudaMalloc/cudaFree may synchronise the device). For them this entry point
// takes its scratch from a fixed array compiled into the library, so it
// allocates nothing at call time.
//
// Costs and rules of the fixed array:
//  * it is ATTN_BWD_NOALLOC_SCRATCH_BYTES (16 MiB) of device memory, held on
//    every GPU on which the library's module is loaded, until the process exits;
//  * every call shares it: two calls that overlap on the GPU (different
//    streams, or different host threads, on the same device) race and corrupt
//    each other; serialise them;
//  * it keeps the previous call's contents; the backward's first kernel
//    re-initialises everything that must start at zero (dQ accumulator, status
//    word), so no clearing is needed between calls.
#include <mutex>

#include "../../include/attn.h"
#include "common.cuh"

namespace {

// Scratch of the no-allocation backward. In host code this name is only a
// host-side stand-in for the device array: its device address must be looked
// up with cudaGetSymbolAddress (done once per device below) before a kernel
// may be given it.
static __device__ __align__(256) unsigned char g_bwd_scratch[ATTN_BWD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Per device: the context the address was looked up in, and the address.
// A device reset (or a destroyed and recreated primary context) reloads the
// module and may move the array, so the address is only reused while the
// current context is the one it was found in.
struct ScratchSlot {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_bwd_scratch on the current device, looked up (with
// that device current) on the first call in each context and cached.
int scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) return ATTN_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (ctx == nullptr || slot.addr == nullptr || slot.ctx != ctx) {
    // The lookup also initialises the device's primary context (and makes it
    // current) when no context is current yet.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr)
      return ATTN_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return ATTN_ERR_CUDA;
    slot.ctx = ctx;
    slot.addr = p;
  }
  *out = slot.addr;
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                int B, int H, int N, int d, int causal, float scale, int dtype,
                                void* stream) {
  const size_t need = attn_bwd_workspace_bytes(B, H, N, d, dtype);
  if (need == 0) {
    // Shape or type rejected: let attn_bwd's checks name the reason.
    return attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, dtype,
                    nullptr, 0, stream);
  }
  if (need > ATTN_BWD_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_INVALID;
  void* scratch = nullptr;
  const int st = scratch_on_current_device(&scratch);
  if (st != ATTN_OK) return st;
  return attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, causal, scale, dtype, scratch,
                  ATTN_BWD_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int attn_bwd_noalloc_last_status(void) {
  void* scratch = nullptr;
  const int st = scratch_on_current_device(&scratch);
  if (st != ATTN_OK) return st;
  return attn_last_status(scratch);
}
