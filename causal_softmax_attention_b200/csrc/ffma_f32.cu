// fp32 forward and backward on the CUDA cores (FFMA), for small fp32 workloads.
//
// Same mathematics as the tensor-core path, entirely in fp32 with expf/logf:
//   forward  S = scale Q K^T (causal filter i >= j), online max-shifted
//            softmax, O = P V, LSE = m + ln z   (ddx issue #217 repro steps;
//            LSE is ddx issue #243 item 2's saved number per row)
//   backward P = exp(S - LSE) recomputed per score, dP = dO V^T,
//            dS = P o (dP - D), dV = P^T dO, dK = scale dS^T Q, dQ = scale dS K
//            (ddx PR #162 "What changed"; shift gradient dropped, issue #243
//            item 1)
//
// Layout of the work: a row (query or key) is owned by TPR = DP/32 threads,
// each holding 32 of its DP (d rounded up to 32/64/128) channels; dot
// products are finished with TPR-wide shuffles. The other side streams
// through shared memory in 32-row tiles. The backward runs two kernels, one
// per key row (dK, dV) and one per query row (dQ), so no atomics are needed
// and the results are deterministic.
#include "common.cuh"

namespace csa {
namespace {

constexpr int kRowsTile = 32;  // rows of the streamed side per shared-memory tile

template <int TPR>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int off = 1; off < TPR; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Loads rows [r0, r0 + 32) x channels [0, DP) of an [N][d] fp32 matrix whose
// rows are `sn` elements apart into shared memory, zero-filling rows >= N and
// channels >= d.
template <int DP>
__device__ __forceinline__ void load_tile(float (*dst)[DP], const float* src, int r0, int N,
                                          int d, long long sn) {
  for (int idx = threadIdx.x; idx < kRowsTile * DP; idx += blockDim.x) {
    const int r = idx / DP, c = idx % DP;
    dst[r][c] = (r0 + r < N && c < d) ? src[(r0 + r) * sn + c] : 0.f;
  }
}

template <int DP>
__global__ void __launch_bounds__(128)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                   const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse,
                   Extent ex, int d, int causal, float scale, RowStrides qs, RowStrides ks,
                   RowStrides os) {
  constexpr int TPR = DP / 32;
  constexpr int R = 128 / TPR;  // rows per block
  __shared__ float sK[kRowsTile][DP];
  __shared__ float sV[kRowsTile][DP];
  const int bh = blockIdx.y;
  const int row = blockIdx.x * R + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const float* qh = q + qs.head(bh);
  const float* kh = k + ks.head(bh);
  const float* vh = v + ks.head(bh);

  float qr[32], acc[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const int ch = 32 * part + c;
    qr[c] = (row < ex.nq && ch < d) ? qh[row * qs.sn + ch] : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, z = 0.f;
  const int last_row = min(ex.nq - 1, blockIdx.x * R + R - 1);
  const int key_end = causal ? min(ex.nk, last_row + ex.q_off + 1) : ex.nk;
  for (int k0 = 0; k0 < key_end; k0 += kRowsTile) {
    __syncthreads();
    load_tile<DP>(sK, kh, k0, ex.nk, d, ks.sn);
    load_tile<DP>(sV, vh, k0, ex.nk, d, ks.sn);
    __syncthreads();
    float s[kRowsTile];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < kRowsTile; ++u) {
      float part_dot = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) part_dot = fmaf(qr[c], sK[u][32 * part + c], part_dot);
      const float dot = group_sum<TPR>(part_dot);
      const int key = k0 + u;
      const bool keep = key < ex.nk && (!causal || key <= row + ex.q_off);
      s[u] = keep ? dot * scale : -INFINITY;
      mx = fmaxf(mx, s[u]);
    }
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;  // nothing kept yet for this row
    const float alpha = expf(m - m_new);
    float zt = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] *= alpha;
#pragma unroll
    for (int u = 0; u < kRowsTile; ++u) {
      const float p = expf(s[u] - m_new);
      zt += p;
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = fmaf(p, sV[u][32 * part + c], acc[c]);
    }
    z = z * alpha + zt;
    m = m_new;
  }
  if (row < ex.nq) {
    const float inv = 1.f / z;
    float* orow = o + os.row(bh, row);
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int ch = 32 * part + c;
      if (ch < d) orow[ch] = acc[c] * inv;
    }
    if (part == 0) lse[static_cast<size_t>(bh) * ex.nq + row] = m + logf(z);
  }
}

// dK, dV: one key row per thread group; query rows stream through shared memory.
template <int DP>
__global__ void __launch_bounds__(128)
    bwd_dkdv_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                        const float* __restrict__ v, const float* __restrict__ dout,
                        const float* __restrict__ lse_pad, const float* __restrict__ d_pad,
                        float* __restrict__ dk, float* __restrict__ dv, Extent ex, int Np, int d,
                        int causal, float scale, RowStrides qs, RowStrides ks, RowStrides os) {
  constexpr int TPR = DP / 32;
  constexpr int R = 128 / TPR;
  __shared__ float sQ[kRowsTile][DP];
  __shared__ float sdO[kRowsTile][DP];
  __shared__ float sL[kRowsTile], sD[kRowsTile];
  const int bh = blockIdx.y;
  const int key = blockIdx.x * R + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const long long off = qs.head(bh), koff = ks.head(bh), ooff = os.head(bh);
  float kr[32], vr[32], gk[32], gv[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const int ch = 32 * part + c;
    const bool in = key < ex.nk && ch < d;
    kr[c] = in ? k[koff + key * ks.sn + ch] : 0.f;
    vr[c] = in ? v[koff + key * ks.sn + ch] : 0.f;
    gk[c] = gv[c] = 0.f;
  }
  // the first query row that can see this block's first key: row + q_off >= key
  const int first_key = blockIdx.x * R;
  const int q_begin = causal ? (max(0, first_key - ex.q_off) / kRowsTile) * kRowsTile : 0;
  for (int q0 = q_begin; q0 < ex.nq; q0 += kRowsTile) {
    __syncthreads();
    load_tile<DP>(sQ, q + off, q0, ex.nq, d, qs.sn);
    load_tile<DP>(sdO, dout + ooff, q0, ex.nq, d, os.sn);
    if (threadIdx.x < kRowsTile) {
      sL[threadIdx.x] = lse_pad[static_cast<size_t>(bh) * Np + q0 + threadIdx.x];
      sD[threadIdx.x] = d_pad[static_cast<size_t>(bh) * Np + q0 + threadIdx.x];
    }
    __syncthreads();
#pragma unroll 4
    for (int u = 0; u < kRowsTile; ++u) {
      const int qi = q0 + u;
      float ps = 0.f, pd = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        ps = fmaf(sQ[u][32 * part + c], kr[c], ps);
        pd = fmaf(sdO[u][32 * part + c], vr[c], pd);
      }
      const float s = group_sum<TPR>(ps) * scale;
      const float dp = group_sum<TPR>(pd);
      const bool keep = qi < ex.nq && key < ex.nk && (!causal || qi + ex.q_off >= key);
      const float p = keep ? expf(s - sL[u]) : 0.f;
      const float ds = p * (dp - sD[u]);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        gv[c] = fmaf(p, sdO[u][32 * part + c], gv[c]);
        gk[c] = fmaf(ds, sQ[u][32 * part + c], gk[c]);
      }
    }
  }
  if (key < ex.nk) {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int ch = 32 * part + c;
      if (ch < d) {
        dk[koff + key * ks.sn + ch] = gk[c] * scale;
        dv[koff + key * ks.sn + ch] = gv[c];
      }
    }
  }
}

// dQ: one query row per thread group; key rows stream through shared memory.
template <int DP>
__global__ void __launch_bounds__(128)
    bwd_dq_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                      const float* __restrict__ v, const float* __restrict__ dout,
                      const float* __restrict__ lse_pad, const float* __restrict__ d_pad,
                      float* __restrict__ dq, Extent ex, int Np, int d, int causal, float scale,
                      RowStrides qs, RowStrides ks, RowStrides os) {
  constexpr int TPR = DP / 32;
  constexpr int R = 128 / TPR;
  __shared__ float sK[kRowsTile][DP];
  __shared__ float sV[kRowsTile][DP];
  const int bh = blockIdx.y;
  const int row = blockIdx.x * R + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const long long off = qs.head(bh), ooff = os.head(bh);
  float qr[32], dor[32], g[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const int ch = 32 * part + c;
    const bool in = row < ex.nq && ch < d;
    qr[c] = in ? q[off + row * qs.sn + ch] : 0.f;
    dor[c] = in ? dout[ooff + row * os.sn + ch] : 0.f;
    g[c] = 0.f;
  }
  const float Li = lse_pad[static_cast<size_t>(bh) * Np + min(row, Np - 1)];
  const float Di = d_pad[static_cast<size_t>(bh) * Np + min(row, Np - 1)];
  const int last_row = min(ex.nq - 1, blockIdx.x * R + R - 1);
  const int key_end = causal ? min(ex.nk, last_row + ex.q_off + 1) : ex.nk;
  for (int k0 = 0; k0 < key_end; k0 += kRowsTile) {
    __syncthreads();
    load_tile<DP>(sK, k + ks.head(bh), k0, ex.nk, d, ks.sn);
    load_tile<DP>(sV, v + ks.head(bh), k0, ex.nk, d, ks.sn);
    __syncthreads();
#pragma unroll 4
    for (int u = 0; u < kRowsTile; ++u) {
      const int key = k0 + u;
      float ps = 0.f, pd = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        ps = fmaf(qr[c], sK[u][32 * part + c], ps);
        pd = fmaf(dor[c], sV[u][32 * part + c], pd);
      }
      const float s = group_sum<TPR>(ps) * scale;
      const float dp = group_sum<TPR>(pd);
      const bool keep = row < ex.nq && key < ex.nk && (!causal || key <= row + ex.q_off);
      const float p = keep ? expf(s - Li) : 0.f;
      const float ds = p * (dp - Di);
#pragma unroll
      for (int c = 0; c < 32; ++c) g[c] = fmaf(ds, sK[u][32 * part + c], g[c]);
    }
  }
  if (row < ex.nq) {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int ch = 32 * part + c;
      if (ch < d) dq[off + row * qs.sn + ch] = g[c] * scale;
    }
  }
}

template <int DP>
cudaError_t fwd_f32_dp(const float* q, const float* k, const float* v, float* o, float* lse,
                       int BH, const Extent& ex, int d, bool causal, float scale,
                       const RowStrides& qs, const RowStrides& ks, const RowStrides& os,
                       cudaStream_t s) {
  constexpr int R = 128 / (DP / 32);
  dim3 grid((ex.nq + R - 1) / R, BH);
  fwd_f32_kernel<DP><<<grid, 128, 0, s>>>(q, k, v, o, lse, ex, d, causal, scale, qs, ks, os);
  return cudaGetLastError();
}

template <int DP>
cudaError_t bwd_f32_dp(const float* q, const float* k, const float* v, const float* dout,
                       float* dq, float* dk, float* dv, int BH, const Extent& ex, int d,
                       bool causal, float scale, const RowStrides& qs, const RowStrides& ks,
                       const RowStrides& os, const Workspace& ws, cudaStream_t s) {
  constexpr int R = 128 / (DP / 32);
  bwd_dkdv_f32_kernel<DP><<<dim3((ex.nk + R - 1) / R, BH), 128, 0, s>>>(
      q, k, v, dout, ws.lse_pad, ws.d_pad, dk, dv, ex, ws.Np, d, causal, scale, qs, ks, os);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_f32_kernel<DP><<<dim3((ex.nq + R - 1) / R, BH), 128, 0, s>>>(
      q, k, v, dout, ws.lse_pad, ws.d_pad, dq, ex, ws.Np, d, causal, scale, qs, ks, os);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int BH, const Extent& ex, int d, bool causal, float scale,
                           const RowStrides& qs, const RowStrides& ks, const RowStrides& os,
                           cudaStream_t s) {
  if (d <= 32) return fwd_f32_dp<32>(q, k, v, o, lse, BH, ex, d, causal, scale, qs, ks, os, s);
  if (d <= 64) return fwd_f32_dp<64>(q, k, v, o, lse, BH, ex, d, causal, scale, qs, ks, os, s);
  return fwd_f32_dp<128>(q, k, v, o, lse, BH, ex, d, causal, scale, qs, ks, os, s);
}

cudaError_t launch_bwd_f32(const float* q, const float* k, const float* v, const float* dout,
                           float* dq, float* dk, float* dv, int BH, const Extent& ex, int d,
                           bool causal, float scale, const RowStrides& qs, const RowStrides& ks,
                           const RowStrides& os, const Workspace& ws, cudaStream_t s) {
  if (d <= 32)
    return bwd_f32_dp<32>(q, k, v, dout, dq, dk, dv, BH, ex, d, causal, scale, qs, ks, os, ws, s);
  if (d <= 64)
    return bwd_f32_dp<64>(q, k, v, dout, dq, dk, dv, BH, ex, d, causal, scale, qs, ks, os, ws, s);
  return bwd_f32_dp<128>(q, k, v, dout, dq, dk, dv, BH, ex, d, causal, scale, qs, ks, os, ws, s);
}

}  // namespace csa
