// Internal declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace csa {

constexpr int kTile = 128;  // rows of a query or key tile on the tensor-core path

constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = -4;

inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Workspace carved out of the caller's buffer for one backward call.
struct Workspace {
  int* status;     // device status word
  float* lse_pad;  // [BH][Np]: LSE (f32 path) or LSE * log2(e) (bf16 path); +inf past N
  float* d_pad;    // [BH][Np]: D_i = sum_c dO_ic O_ic; 0 past N
  float* dq_acc;   // [BH][Np][d] fp32 dQ accumulator (bf16 path only)
  int Np;          // N rounded up to whole 128-row tiles
};

struct WorkspaceLayout {
  size_t status_off, lse_off, d_off, dq_off, total;
  int Np;
};

WorkspaceLayout workspace_layout(int B, int H, int N, int d, int dtype);
Workspace carve_workspace(void* base, const WorkspaceLayout& L);

// Limit of one device-side bounded wait, in SM clock cycles (about 1.1 s at
// 1.9 GHz; a healthy wait lasts microseconds).
constexpr uint64_t kWaitLimitCycles = 1ull << 31;

// ---- launchers (return cudaError_t from the launch) ----
cudaError_t launch_preprocess(const void* o, const void* dout, const float* lse, int BH, int N,
                              int d, bool bf16, const Workspace& ws, cudaStream_t s);
cudaError_t launch_dq_convert(void* dq, int BH, int N, int d, float scale, const Workspace& ws,
                              cudaStream_t s);
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int BH, int N, int d, bool causal, float scale, cudaStream_t s);
cudaError_t launch_bwd_f32(const float* q, const float* k, const float* v, const float* dout,
                           float* dq, float* dk, float* dv, int BH, int N, int d, bool causal,
                           float scale, const Workspace& ws, cudaStream_t s);

// Tensor-core (tcgen05) path; tensor maps are encoded by the caller.
struct TmaMaps {
  CUtensorMap a, b, c, d;
};
// block_mask: device [T][T] tile kinds (0 none, 1 all, 2 key <= query inside
// the tile), T = ceil(N / 128), or null for the causal / full filter.
cudaError_t launch_fwd_bf16(const TmaMaps& maps, void* o, float* lse, int* status, int BH, int N,
                            int d, bool causal, float scale, const uint8_t* block_mask,
                            cudaStream_t s);
cudaError_t launch_bwd_bf16(const TmaMaps& maps, const Workspace& ws, void* dk, void* dv, int BH,
                            int N, int d, bool causal, float scale, uint64_t wait_limit_cycles,
                            int inject_fault, const uint8_t* block_mask, cudaStream_t s);

int* fwd_status_ptr();  // library-owned forward status word on the current device

}  // namespace csa
