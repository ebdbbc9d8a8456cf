// C ABI of the library (declared in include/attn.h): argument checks, the
// workspace layout, TMA tensor-map encoding and kernel dispatch. Everything
// is enqueued on the caller's stream; nothing here allocates device memory.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "common.cuh"

namespace csa {

WorkspaceLayout workspace_layout(int B, int H, int N, int d, int dtype) {
  WorkspaceLayout L{};
  const size_t BH = static_cast<size_t>(B) * H;
  L.Np = round_up(N, kTile);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  L.status_off = 0;
  L.lse_off = 256;
  L.d_off = L.lse_off + up(BH * L.Np * sizeof(float));
  L.dq_off = L.d_off + up(BH * L.Np * sizeof(float));
  L.total = L.dq_off + (dtype == ATTN_BF16 ? up(BH * L.Np * d * sizeof(float)) : 0);
  return L;
}

Workspace carve_workspace(void* base, const WorkspaceLayout& L) {
  char* b = static_cast<char*>(base);
  Workspace w;
  w.status = reinterpret_cast<int*>(b + L.status_off);
  w.lse_pad = reinterpret_cast<float*>(b + L.lse_off);
  w.d_pad = reinterpret_cast<float*>(b + L.d_off);
  w.dq_acc = reinterpret_cast<float*>(b + L.dq_off);
  w.Np = L.Np;
  return w;
}

}  // namespace csa

namespace {

using namespace csa;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape / pointer checks shared by every entry point.
int check_shape(int B, int H, int N, int d, int dtype) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return ATTN_ERR_INVALID;
  if (dtype != ATTN_F32 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (dtype == ATTN_BF16 && d != 32 && d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (dtype == ATTN_F32 && d > 128) return ATTN_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  const long long T = (static_cast<long long>(N) + kTile - 1) / kTile;
  if (BH > (1LL << 30) || BH * T > 0x7fffffffLL) return ATTN_ERR_INVALID;
  return ATTN_OK;
}

// Extents of a rectangular call: at least one query row and one key, a
// query offset in [0, 2^30], and tile counts the launch grids can hold.
int check_extent(int B, int H, const Extent& ex, int d, int dtype) {
  int st = check_shape(B, H, ex.nq, d, dtype);
  if (st != ATTN_OK) return st;
  if ((st = check_shape(B, H, ex.nk, d, dtype)) != ATTN_OK) return st;
  if (ex.q_off < 0 || ex.q_off > (1 << 30)) return ATTN_ERR_INVALID;
  return ATTN_OK;
}

Extent square(int N) { return {N, N, 0}; }

bool all_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p == nullptr || !aligned16(p)) return false;
  return true;
}

// Tensor pointers: 16-byte aligned for bf16 (tensor maps, vector access),
// 4-byte aligned for fp32 (the FFMA kernels read single elements).
bool tensors_aligned(int dtype, std::initializer_list<const void*> ps) {
  const uintptr_t mask = dtype == ATTN_BF16 ? 15u : 3u;
  for (const void* p : ps)
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & mask) != 0) return false;
  return true;
}

// The tensor-core kernels are built for sm_100a only.
int check_device_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return (major == 10 && minor == 0) ? ATTN_OK : ATTN_ERR_CUDA;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D map {d, N, H, B} over a bf16 array whose rows `rs` lays out: box =
// `box_rows` rows (a tile, or the backward-over-backward's 64-row halves) x
// min(d, 64) channels of one (b, h), swizzled to match the UMMA canonical
// layout. Rows past N read as zero.
bool make_map(CUtensorMap* m, const void* base, int B, int N, int d, const RowStrides& rs,
              int box_rows = kTile) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int ch = d >= 64 ? 64 : d;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(rs.H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(rs.sn) * 2, static_cast<cuuint64_t>(rs.sh) * 2,
                           static_cast<cuuint64_t>(rs.sb) * 2};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(ch), static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapSwizzle swz =
      ch * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Strides from the caller: positive, rows of one head at least d apart, and
// for bf16 whole 16-byte units (the tensor maps and the vector stores need
// it); below the tensor maps' 2^40-byte stride limit.
int check_strides(const long long* st, int H, int d, int dtype, RowStrides* out) {
  if (st == nullptr) return ATTN_ERR_INVALID;
  const long long lim = 1LL << 36;
  for (int i = 0; i < 3; ++i)
    if (st[i] <= 0 || st[i] >= lim) return ATTN_ERR_INVALID;
  if (st[2] < d) return ATTN_ERR_INVALID;
  if (dtype == ATTN_BF16)
    for (int i = 0; i < 3; ++i)
      if (st[i] % 8 != 0) return ATTN_ERR_INVALID;
  *out = {st[0], st[1], st[2], H};
  return ATTN_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA; }

// Debug builds fill an output with NaN (all-ones bytes: NaN in bf16 and in
// fp32) before the kernels run, stream-ordered, so that an element no kernel
// writes shows up; release builds do nothing. Only contiguous outputs are
// filled (a strided view's rows need not tile its span).
bool is_dense(const RowStrides& rs, int n, int d) {
  return rs.sn == d && rs.sh == static_cast<long long>(n) * d && rs.sb == rs.sh * rs.H;
}

int poison(void* p, size_t elems, size_t elem_bytes, cudaStream_t s) {
#ifdef ATTN_DEBUG
  if (p != nullptr && elems > 0)
    return from_cuda(cudaMemsetAsync(p, 0xFF, elems * elem_bytes, s));
#else
  (void)p, (void)elems, (void)elem_bytes, (void)s;
#endif
  return ATTN_OK;
}

struct FaultInjection {
  int armed = 0;
  unsigned long long limit_cycles = 0;
};
FaultInjection g_fault;
std::mutex g_fault_mu;

int check_ws(int B, int H, int N, int d, int dtype, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned16(ws)) return ATTN_ERR_INVALID;
  if (ws_bytes < workspace_layout(B, H, N, d, dtype).total) return ATTN_ERR_INVALID;
  return ATTN_OK;
}

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported dtype / head dimension";
    case ATTN_ERR_CUDA: return "CUDA error (launch failed or device is not sm_100)";
    case ATTN_ERR_TIMEOUT: return "device-side wait timed out";
    case ATTN_ERR_BOUNDS: return "device-side bounds check failed (debug build)";
    default: return "unknown status";
  }
}

size_t attn_bwd_workspace_bytes(int B, int H, int N, int d, int dtype) {
  if (check_shape(B, H, N, d, dtype) != ATTN_OK) return 0;
  return workspace_layout(B, H, N, d, dtype).total;
}

namespace {

// Every implementation takes the row strides of q, k, v (and of dq, dk, dv:
// qs) and of o, dout (os); the plain entry points pass the contiguous layout.
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             const Extent& ex, int d, int causal, float scale, int dtype, const uint8_t* bmask,
             const RowStrides& qs, const RowStrides& os, void* stream, const RowStrides& ks) {
  if (!tensors_aligned(dtype, {q, k, v, o}) || !all_aligned({lse})) return ATTN_ERR_INVALID;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID;
  int st = check_extent(B, H, ex, d, dtype);
  if (st != ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (dtype == ATTN_BF16 && (st = check_device_sm100()) != ATTN_OK) return st;
  if (is_dense(os, ex.nq, d) &&
      (poison(o, static_cast<size_t>(BH) * ex.nq * d, dtype == ATTN_BF16 ? 2 : 4, s) != ATTN_OK ||
       poison(lse, static_cast<size_t>(BH) * ex.nq, 4, s) != ATTN_OK))
    return ATTN_ERR_CUDA;
  if (dtype == ATTN_F32)
    return from_cuda(launch_fwd_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                    static_cast<const float*>(v), static_cast<float*>(o), lse, BH,
                                    ex, d, causal != 0, scale, qs, ks, os, s));
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  TmaMaps m;
  if (!make_map(&m.a, q, B, ex.nq, d, qs) || !make_map(&m.b, k, B, ex.nk, d, ks) ||
      !make_map(&m.c, v, B, ex.nk, d, ks))
    return ATTN_ERR_CUDA;
  int* status = fwd_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  return from_cuda(
      launch_fwd_bf16(m, o, lse, status, BH, ex, d, causal != 0, scale, bmask, os, s));
}

int preprocess_impl(const void* o, const void* dout, const float* lse, int B, int H, int N, int d,
                    int dtype, void* workspace, size_t workspace_bytes, const RowStrides& os,
                    void* stream) {
  if (!tensors_aligned(dtype, {o, dout}) || !all_aligned({lse})) return ATTN_ERR_INVALID;
  int st = check_shape(B, H, N, d, dtype);
  if (st != ATTN_OK) return st;
  if ((st = check_ws(B, H, N, d, dtype, workspace, workspace_bytes)) != ATTN_OK) return st;
  const Workspace ws = carve_workspace(workspace, workspace_layout(B, H, N, d, dtype));
  return from_cuda(launch_preprocess(o, dout, lse, B * H, N, d, dtype == ATTN_BF16, os, ws,
                                     static_cast<cudaStream_t>(stream)));
}

int bwd_main_impl(const void* q, const void* k, const void* v, const void* dout, void* dq,
                  void* dk, void* dv, int B, int H, const Extent& ex, int d, int causal,
                  float scale, int dtype, void* workspace, size_t workspace_bytes,
                  const uint8_t* bmask, const RowStrides& qs, const RowStrides& os,
                  void* stream, const RowStrides& ks) {
  if (!tensors_aligned(dtype, {q, k, v, dout, dq, dk, dv})) return ATTN_ERR_INVALID;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID;
  int st = check_extent(B, H, ex, d, dtype);
  if (st != ATTN_OK) return st;
  if ((st = check_ws(B, H, ex.nq, d, dtype, workspace, workspace_bytes)) != ATTN_OK) return st;
  const Workspace ws = carve_workspace(workspace, workspace_layout(B, H, ex.nq, d, dtype));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (dtype == ATTN_F32)
    return from_cuda(launch_bwd_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                    static_cast<const float*>(v),
                                    static_cast<const float*>(dout), static_cast<float*>(dq),
                                    static_cast<float*>(dk), static_cast<float*>(dv), BH, ex, d,
                                    causal != 0, scale, qs, ks, os, ws, s));
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  TmaMaps m;
  if (!make_map(&m.a, q, B, ex.nq, d, qs) || !make_map(&m.b, k, B, ex.nk, d, ks) ||
      !make_map(&m.c, v, B, ex.nk, d, ks) || !make_map(&m.d, dout, B, ex.nq, d, os))
    return ATTN_ERR_CUDA;
  int inject = 0;
  unsigned long long limit = kWaitLimitCycles;
  {
    std::lock_guard<std::mutex> g(g_fault_mu);
    if (g_fault.armed) {
      inject = 1;
      limit = g_fault.limit_cycles;
      g_fault.armed = 0;
    }
  }
  return from_cuda(launch_bwd_bf16(m, ws, dk, dv, BH, ex, d, causal != 0, scale, limit, inject,
                                   bmask, ks, s));
}

int dq_convert_impl(void* dq, int B, int H, int N, int d, float scale, int dtype,
                    void* workspace, size_t workspace_bytes, const RowStrides& qs, void* stream) {
  if (!tensors_aligned(dtype, {dq})) return ATTN_ERR_INVALID;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID;
  int st = check_shape(B, H, N, d, dtype);
  if (st != ATTN_OK) return st;
  if ((st = check_ws(B, H, N, d, dtype, workspace, workspace_bytes)) != ATTN_OK) return st;
  if (dtype == ATTN_F32) return ATTN_OK;
  const Workspace ws = carve_workspace(workspace, workspace_layout(B, H, N, d, dtype));
  return from_cuda(
      launch_dq_convert(dq, B * H, N, d, scale, qs, ws, static_cast<cudaStream_t>(stream)));
}

// The whole backward: every argument is checked before the first launch, so
// a bad call enqueues nothing.
int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int H, const Extent& ex,
             int d, int causal, float scale, int dtype, void* workspace, size_t workspace_bytes,
             const uint8_t* bmask, const RowStrides& qs, const RowStrides& os, void* stream,
             const RowStrides& ks) {
  if (!tensors_aligned(dtype, {q, k, v, o, dout, dq, dk, dv}) || !all_aligned({lse}))
    return ATTN_ERR_INVALID;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID;
  int st = check_extent(B, H, ex, d, dtype);
  if (st != ATTN_OK) return st;
  if (bmask != nullptr && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if ((st = check_ws(B, H, ex.nq, d, dtype, workspace, workspace_bytes)) != ATTN_OK) return st;
  if (dtype == ATTN_BF16 && (st = check_device_sm100()) != ATTN_OK) return st;
  {
    const size_t bh = static_cast<size_t>(B) * H, eb = dtype == ATTN_BF16 ? 2 : 4;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((is_dense(qs, ex.nq, d) && poison(dq, bh * ex.nq * d, eb, s) != ATTN_OK) ||
        (is_dense(ks, ex.nk, d) && (poison(dk, bh * ex.nk * d, eb, s) != ATTN_OK ||
                                    poison(dv, bh * ex.nk * d, eb, s) != ATTN_OK)))
      return ATTN_ERR_CUDA;
  }
  st = preprocess_impl(o, dout, lse, B, H, ex.nq, d, dtype, workspace, workspace_bytes, os,
                       stream);
  if (st != ATTN_OK) return st;
  st = bwd_main_impl(q, k, v, dout, dq, dk, dv, B, H, ex, d, causal, scale, dtype, workspace,
                     workspace_bytes, bmask, qs, os, stream, ks);
  if (st != ATTN_OK) return st;
  return dq_convert_impl(dq, B, H, ex.nq, d, scale, dtype, workspace, workspace_bytes, qs,
                         stream);
}

RowStrides dense(int H, int N, int d) { return contiguous_strides(H, N, d); }

}  // namespace

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int N, int d, int causal, float scale, int dtype, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, H, square(N), d, causal, scale, dtype, nullptr, dense(H, N, d),
                  dense(H, N, d), stream, dense(H, N, d));
}

int attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int N, int d, const unsigned char* block_mask, float scale, int dtype,
                    void* stream) {
  if (block_mask == nullptr) return ATTN_ERR_INVALID;
  if (dtype != ATTN_BF16) return check_shape(B, H, N, d, dtype) == ATTN_OK ? ATTN_ERR_UNSUPPORTED
                                                                         : ATTN_ERR_INVALID;
  return fwd_impl(q, k, v, o, lse, B, H, square(N), d, 0, scale, dtype, block_mask, dense(H, N, d),
                  dense(H, N, d), stream, dense(H, N, d));
}

int attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, const long long* qkv_strides,
                     const long long* o_strides, int causal, float scale, int dtype,
                     void* stream) {
  RowStrides qs{}, os{};
  int st = check_shape(B, H, N, d, dtype);
  if (st != ATTN_OK) return st;
  if ((st = check_strides(qkv_strides, H, d, dtype, &qs)) != ATTN_OK) return st;
  if ((st = check_strides(o_strides, H, d, dtype, &os)) != ATTN_OK) return st;
  return fwd_impl(q, k, v, o, lse, B, H, square(N), d, causal, scale, dtype, nullptr, qs, os, stream, qs);
}

int attn_bwd_preprocess(const void* o, const void* dout, const float* lse, int B, int H, int N,
                        int d, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return preprocess_impl(o, dout, lse, B, H, N, d, dtype, workspace, workspace_bytes,
                         dense(H, N, d), stream);
}

int attn_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dq,
                  void* dk, void* dv, int B, int H, int N, int d, int causal, float scale,
                  int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_main_impl(q, k, v, dout, dq, dk, dv, B, H, square(N), d, causal, scale, dtype, workspace,
                       workspace_bytes, nullptr, dense(H, N, d), dense(H, N, d), stream, dense(H, N, d));
}

int attn_bwd_main_masked(const void* q, const void* k, const void* v, const void* dout, void* dq,
                         void* dk, void* dv, int B, int H, int N, int d,
                         const unsigned char* block_mask, float scale, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (block_mask == nullptr || !all_aligned({q, k, v, dout, dq, dk, dv})) return ATTN_ERR_INVALID;
  const int st = check_shape(B, H, N, d, dtype);
  if (st != ATTN_OK) return st;
  if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  return bwd_main_impl(q, k, v, dout, dq, dk, dv, B, H, square(N), d, 0, scale, dtype, workspace,
                       workspace_bytes, block_mask, dense(H, N, d), dense(H, N, d), stream, dense(H, N, d));
}

int attn_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, int dtype,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return dq_convert_impl(dq, B, H, N, d, scale, dtype, workspace, workspace_bytes, dense(H, N, d),
                         stream);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
             int causal, float scale, int dtype, void* workspace, size_t workspace_bytes,
             void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, square(N), d, causal, scale, dtype, workspace,
                  workspace_bytes, nullptr, dense(H, N, d), dense(H, N, d), stream, dense(H, N, d));
}

int attn_bwd_masked(const void* q, const void* k, const void* v, const void* o,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                    int H, int N, int d, const unsigned char* block_mask, float scale, int dtype,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (block_mask == nullptr) return ATTN_ERR_INVALID;
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, square(N), d, 0, scale, dtype, workspace,
                  workspace_bytes, block_mask, dense(H, N, d), dense(H, N, d), stream, dense(H, N, d));
}

int attn_bwd_strided(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                     int H, int N, int d, const long long* qkv_strides,
                     const long long* o_strides, int causal, float scale, int dtype,
                     void* workspace, size_t workspace_bytes, void* stream) {
  RowStrides qs{}, os{};
  int st = check_shape(B, H, N, d, dtype);
  if (st != ATTN_OK) return st;
  if ((st = check_strides(qkv_strides, H, d, dtype, &qs)) != ATTN_OK) return st;
  if ((st = check_strides(o_strides, H, d, dtype, &os)) != ATTN_OK) return st;
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, square(N), d, causal, scale, dtype, workspace,
                  workspace_bytes, nullptr, qs, os, stream, qs);
}

int attn_fwd_rect(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int H, int n_q, int n_k, int d, int q_offset, int causal, float scale,
                  int dtype, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, H, Extent{n_q, n_k, q_offset}, d, causal, scale, dtype,
                  nullptr, dense(H, n_q, d), dense(H, n_q, d), stream, dense(H, n_k, d));
}

int attn_bwd_rect(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int H, int n_q, int n_k,
                  int d, int q_offset, int causal, float scale, int dtype, void* workspace,
                  size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, Extent{n_q, n_k, q_offset}, d, causal,
                  scale, dtype, workspace, workspace_bytes, nullptr, dense(H, n_q, d),
                  dense(H, n_q, d), stream, dense(H, n_k, d));
}

// Backward-over-backward: the f32 backward's workspace (status, padded LSE,
// D) followed by the two row scalars r and g, [BH][Np] floats each.
namespace {
size_t bob_extra_off(int B, int H, int N, int d) {
  return (workspace_layout(B, H, N, d, ATTN_F32).total + 255) / 256 * 256;
}
}  // namespace

// (the same for both dtypes: the bf16 path has no dQ accumulator)
size_t attn_bwd_bwd_workspace_bytes(int B, int H, int N, int d, int dtype) {
  if (check_shape(B, H, N, d, dtype) != ATTN_OK) return 0;
  const size_t rows = static_cast<size_t>(B) * H * round_up(N, kTile);
  return bob_extra_off(B, H, N, d) + 2 * ((rows * sizeof(float) + 255) / 256 * 256);
}

int attn_bwd_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, const void* uq, const void* uk, const void* uv, void* gq,
                 void* gk, void* gv, void* gdout, int B, int H, int N, int d, int causal,
                 float scale, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (!tensors_aligned(dtype, {q, k, v, o, dout, uq, uk, uv, gq, gk, gv, gdout}) ||
      !all_aligned({lse}))
    return ATTN_ERR_INVALID;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID;
  int st = check_shape(B, H, N, d, dtype);
  if (st != ATTN_OK) return st;
  if (workspace == nullptr || !aligned16(workspace) ||
      workspace_bytes < attn_bwd_bwd_workspace_bytes(B, H, N, d, dtype))
    return ATTN_ERR_INVALID;
  {
    const size_t n = static_cast<size_t>(B) * H * N * d, eb = dtype == ATTN_BF16 ? 2 : 4;
    for (void* out : {gq, gk, gv, gdout})
      if (poison(out, n, eb, static_cast<cudaStream_t>(stream)) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  const size_t rows = static_cast<size_t>(B) * H * round_up(N, kTile);
  float* r_pad = reinterpret_cast<float*>(static_cast<char*>(workspace) + bob_extra_off(B, H, N, d));
  float* g_pad =
      reinterpret_cast<float*>(reinterpret_cast<char*>(r_pad) + (rows * sizeof(float) + 255) / 256 * 256);
  if (dtype == ATTN_BF16) {
    if ((st = check_device_sm100()) != ATTN_OK) return st;
    // the bf16 preprocess (D, -LSE log2 e) into the f32 layout: no dQ accumulator
    Workspace ws = carve_workspace(workspace, workspace_layout(B, H, N, d, ATTN_F32));
    ws.dq_acc = nullptr;
    const RowStrides rs = dense(H, N, d);
    CUtensorMap maps[7];
    const void* src[7] = {q, k, v, dout, uq, uk, uv};
    for (int i = 0; i < 7; ++i)
      if (!make_map(&maps[i], src[i], B, N, d, rs, kBobBoxRows)) return ATTN_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = from_cuda(launch_preprocess(o, dout, lse, B * H, N, d, true, rs, ws, s));
    if (st != ATTN_OK) return st;
    int inject = 0;
    unsigned long long limit = kWaitLimitCycles;
    {
      std::lock_guard<std::mutex> g(g_fault_mu);
      if (g_fault.armed) {
        inject = 1;
        limit = g_fault.limit_cycles;
        g_fault.armed = 0;
      }
    }
    return from_cuda(launch_bob_bf16(maps, src, ws, r_pad, g_pad, gq, gk, gv, gdout, B * H, H, N, d,
                                     causal != 0, scale, limit, inject, s));
  }
  st = preprocess_impl(o, dout, lse, B, H, N, d, dtype, workspace, workspace_bytes,
                       dense(H, N, d), stream);
  if (st != ATTN_OK) return st;
  const Workspace ws = carve_workspace(workspace, workspace_layout(B, H, N, d, dtype));
  return from_cuda(launch_bob_f32(
      static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
      static_cast<const float*>(dout), static_cast<const float*>(uq),
      static_cast<const float*>(uk), static_cast<const float*>(uv), static_cast<float*>(gq),
      static_cast<float*>(gk), static_cast<float*>(gv), static_cast<float*>(gdout), B * H, N, d,
      causal != 0, scale, ws, r_pad, g_pad, static_cast<cudaStream_t>(stream)));
}

int attn_last_status(const void* workspace) {
  if (workspace == nullptr) return ATTN_ERR_INVALID;
  int v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return v;
}

int attn_fwd_last_status(void) {
  int* p = fwd_status_ptr();
  if (!p) return ATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return v;
}

int attn_test_exp2(const float* x, float* poly, float* mufu, int n, void* stream) {
  if (x == nullptr || poly == nullptr || mufu == nullptr || n < 0) return ATTN_ERR_INVALID;
  if (n == 0) return ATTN_OK;
  return from_cuda(launch_exp2_pair(x, poly, mufu, n, static_cast<cudaStream_t>(stream)));
}

int attn_test_arm_timeout(unsigned long long wait_limit_cycles) {
  if (wait_limit_cycles == 0) return ATTN_ERR_INVALID;
  std::lock_guard<std::mutex> g(g_fault_mu);
  g_fault.armed = 1;
  g_fault.limit_cycles = wait_limit_cycles;
  return ATTN_OK;
}

}  // extern "C"
