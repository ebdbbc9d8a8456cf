// Internal declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace csa {

constexpr int kTile = 128;  // rows of a query or key tile on the tensor-core path
constexpr int kBobBoxRows = 64;  // rows of one backward-over-backward TMA box (half a tile)

constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = -4;
constexpr int kStatusBounds = -5;  // a device-side bounds check of a debug build failed

// Debug builds (compiled with ATTN_DEBUG) check tile coordinates and row
// indices before the global accesses a thread makes; a failed check writes
// kStatusBounds into the call's status word and the access is skipped or
// redirected to a valid tile -- never a trap. Release builds compile the
// checks away (the condition is not even evaluated).
#ifdef ATTN_DEBUG
#define CSA_IN_BOUNDS(cond, status) ((cond) ? true : (atomicExch((status), kStatusBounds), false))
#else
#define CSA_IN_BOUNDS(cond, status) true
#endif

inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Element strides of a [B][H][N][d] view whose channel stride is 1: row i of
// head (b, h) starts at element b*sb + h*sh + i*sn. H splits a flat head
// index bh = b*H + h. The contiguous layout is {H*N*d, N*d, d}; the
// (sequence, position, head, channel) tables of ddx issue #217 are
// {N*H*d, d, H*d}.
struct RowStrides {
  long long sb, sh, sn;
  int H;
  __host__ __device__ __forceinline__ long long head(int bh) const {
    return static_cast<long long>(bh / H) * sb + static_cast<long long>(bh % H) * sh;
  }
  __host__ __device__ __forceinline__ long long row(int bh, int i) const {
    return head(bh) + static_cast<long long>(i) * sn;
  }
};
inline RowStrides contiguous_strides(int H, int N, int d) {
  return {static_cast<long long>(H) * N * d, static_cast<long long>(N) * d, d, H};
}

// Workspace carved out of the caller's buffer for one backward call.
struct Workspace {
  int* status;     // device status word
  float* lse_pad;  // [BH][Np]: LSE, +inf past N (f32 path); -LSE * log2(e), -inf past N (bf16)
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
// qs: strides of q, k, v and of dq, dk, dv; os: strides of o and dout.
cudaError_t launch_preprocess(const void* o, const void* dout, const float* lse, int BH, int N,
                              int d, bool bf16, const RowStrides& os, const Workspace& ws,
                              cudaStream_t s);
cudaError_t launch_dq_convert(void* dq, int BH, int N, int d, float scale, const RowStrides& qs,
                              const Workspace& ws, cudaStream_t s);
// Query and key extents of a head: N_q query rows, N_k keys; query row r
// stands for position q_off + r and key j for position j, and the causal
// filter keeps a score when the query's position is at least the key's. The
// square problem is {N, N, 0}.
struct Extent {
  int nq, nk, q_off;
};

// qs: strides of q and dq; ks: of k, v, dk, dv; os: of o and dout.
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int BH, const Extent& ex, int d, bool causal, float scale,
                           const RowStrides& qs, const RowStrides& ks, const RowStrides& os,
                           cudaStream_t s);
cudaError_t launch_bwd_f32(const float* q, const float* k, const float* v, const float* dout,
                           float* dq, float* dk, float* dv, int BH, const Extent& ex, int d,
                           bool causal, float scale, const RowStrides& qs, const RowStrides& ks,
                           const RowStrides& os, const Workspace& ws, cudaStream_t s);

// Backward-over-backward on the CUDA cores (contiguous fp32 [BH][N][d]);
// needs the preprocess's lse_pad and d_pad in `ws`, and writes the two row
// scalars to r_pad, g_pad ([BH][Np] each).
cudaError_t launch_bob_f32(const float* q, const float* k, const float* v, const float* dout,
                           const float* uq, const float* uk, const float* uv, float* gq,
                           float* gk, float* gv, float* gdout, int BH, int N, int d, bool causal,
                           float scale, const Workspace& ws, float* r_pad, float* g_pad,
                           cudaStream_t s);

// Tensor-core (tcgen05) path; tensor maps are encoded by the caller, each a
// 4-D map {d, N, H, B} with a box of {min(d, 64), 128, 1, 1}, loaded at
// coordinates {channel, row, h, b}.
struct TmaMaps {
  CUtensorMap a, b, c, d;
};
// block_mask: device [T][T] tile kinds (0 none, 1 all, 2 key <= query inside
// the tile), T = ceil(N / 128), or null for the causal / full filter.
// (q and o have ex.nq rows per head, k and v ex.nk; a block mask is square,
// ex.nq == ex.nk, q_off == 0)
cudaError_t launch_fwd_bf16(const TmaMaps& maps, void* o, float* lse, int* status, int BH,
                            const Extent& ex, int d, bool causal, float scale,
                            const uint8_t* block_mask, const RowStrides& os, cudaStream_t s);
cudaError_t launch_bwd_bf16(const TmaMaps& maps, const Workspace& ws, void* dk, void* dv, int BH,
                            const Extent& ex, int d, bool causal, float scale,
                            uint64_t wait_limit_cycles, int inject_fault,
                            const uint8_t* block_mask, const RowStrides& ks, cudaStream_t s);

// Backward-over-backward on the tensor cores (bf16, d in {32, 64, 128}):
// maps = {q, k, v, dout, uq, uk, uv} as for the tensor-core backward (4-D,
// contiguous [B][H][N][d]); needs the bf16 preprocess's lse_pad and d_pad in
// `ws`, and writes the two row scalars to r_pad, g_pad ([BH][Np] each).
// maps and src: q, k, v, dout, uq, uk, uv (contiguous [BH][N][d] bf16)
// wait_limit_cycles bounds every device wait; inject_fault withholds the rows
// kernel's first score signal (the timeout test's hook)
cudaError_t launch_bob_bf16(const CUtensorMap (&maps)[7], const void* const (&src)[7],
                            const Workspace& ws, float* r_pad, float* g_pad, void* gq, void* gk,
                            void* gv, void* gdo, int BH, int H, int N, int d, bool causal,
                            float scale, uint64_t wait_limit_cycles, int inject_fault,
                            cudaStream_t s);

int* fwd_status_ptr();  // library-owned forward status word on the current device

// Test hook: 2^x by the forward's FMA-pipe polynomial and by MUFU ex2.approx.
cudaError_t launch_exp2_pair(const float* x, float* poly, float* mufu, int n, cudaStream_t s);

}  // namespace csa
