// Backward-over-backward of causal softmax attention on the CUDA cores
// (fp32 FFMA): the gradient of L2 = <U_Q, dQ> + <U_K, dK> + <U_V, dV> with
// respect to Q, K, V and dO, where (dQ, dK, dV) is attention's first
// backward. The operation and its shape -- two row-wise scalars, then affine
// maps of recomputed tiles, in two passes over the scores -- follow the
// FlashBoB listing ("Approaching I/O-optimality for Approximate Attention",
// abstract). Per score pair (i, j), recomputed from the rows alone:
//
//   P  = exp(s q_i.k_j - LSE_i)         dP = dO_i.v_j
//   M  = s (u_Q,i . k_j + q_i . u_K,j)  W  = dO_i . u_V,j
//   row scalars  r_i = sum_j P M,  g_i = sum_j P (M dP) - 2 r_i D_i + sum_j P W
//   dS = P (dP - D_i)   E = P (M - r_i)   dS2 = P (M (dP - D_i) - r_i dP + W - g_i)
//
//   gQ_i  = s sum_j (dS u_K,j + dS2 k_j)     gdO_i = sum_j (E v_j + P u_V,j)
//   gK_j  = s sum_i (dS u_Q,i + dS2 q_i)     gV_j  = sum_i E dO_i
//
// (D_i = sum_c dO_ic O_ic from the first backward's preprocess.) Kernel 1
// owns query rows: one sweep over the key tiles accumulates r, g and seven
// vectors that gQ and gdO are affine combinations of (in r and g), and r, g
// go to the workspace. Kernel 2 owns key rows and accumulates gK and gV over
// the query tiles. No atomics: the
// results are deterministic. Each thread holds CPT channels of its row's
// vectors (16, or 8 at d = 128 and for small problems, where twice the CTAs
// and ~105 instead of ~166 registers win); TPR = DP/CPT threads share a row
// and finish dot products with shuffles, the other side streams through
// shared memory 16 rows at a time.
#include "common.cuh"

namespace csa {
namespace {

constexpr int kRows = 16;  // rows of the streamed side per shared-memory tile

template <int TPR>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int off = 1; off < TPR; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// rows [r0, r0 + kRows) x channels [0, DP) of an [N][d] fp32 head (rows d
// apart) into shared memory; rows >= N and channels >= d read as zero
template <int DP>
__device__ __forceinline__ void stage(float (*dst)[DP], const float* src, int r0, int N, int d) {
  for (int idx = threadIdx.x; idx < kRows * DP; idx += blockDim.x) {
    const int r = idx / DP, c = idx % DP;
    dst[r][c] = (r0 + r < N && c < d) ? src[static_cast<size_t>(r0 + r) * d + c] : 0.f;
  }
}

template <int CPT>
__device__ __forceinline__ void load_row(float (&dst)[CPT], const float* src, int row, int N,
                                         int d, int part) {
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int ch = CPT * part + c;
    dst[c] = (row < N && ch < d) ? src[static_cast<size_t>(row) * d + ch] : 0.f;
  }
}

// four independent partial sums: the chains are a quarter as long, so the
// latency of one dot product no longer serialises the pair
template <int DP, int CPT>
__device__ __forceinline__ float dot(const float (&a)[CPT], const float (*tile)[DP], int u,
                                     int part) {
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < CPT; ++c) s[c % 4] = fmaf(a[c], tile[u][CPT * part + c], s[c % 4]);
  return (s[0] + s[1]) + (s[2] + s[3]);
}

template <int CPT>
__device__ __forceinline__ void store_row(float* dst, const float (&a)[CPT], float mul, int row,
                                          int N, int d, int part) {
  if (row >= N) return;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int ch = CPT * part + c;
    if (ch < d) dst[static_cast<size_t>(row) * d + ch] = a[c] * mul;
  }
}

struct BobArgs {
  const float *q, *k, *v, *dout, *uq, *uk, *uv;
  float *gq, *gk, *gv, *gdout;
  const float *lse_pad, *d_pad;  // [BH][Np]: LSE (+inf past N), D (0 past N)
  float *r_pad, *g_pad;          // [BH][Np]: the two row scalars (0 past N)
  int N, Np, d, causal;
  float scale;
};

// ------------------------------------------------------------ query rows
// One sweep over the key tiles. dS2 needs the complete row scalar g, so
// instead of a second sweep the row side is kept affine in (r, g): with
// per-pair scalars p, dP, M, W,
//   gQ / s = sum p (dP - D) u_K + sum p (M (dP - D) + W) k - r sum p dP k - g sum p k
//   gdO    = sum p M v - r sum p v + sum p u_V
// so seven vectors are accumulated and combined once r and g are known.
template <int DP, int CPT>
__global__ void __launch_bounds__(128) bob_rows_f32_kernel(const BobArgs a) {
  constexpr int TPR = DP / CPT;
  constexpr int R = 128 / TPR;
  __shared__ float sK[kRows][DP], sV[kRows][DP], sUK[kRows][DP], sUV[kRows][DP];
  const int bh = blockIdx.y;
  const int row = blockIdx.x * R + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const size_t off = static_cast<size_t>(bh) * a.N * a.d;
  const float *kh = a.k + off, *vh = a.v + off, *ukh = a.uk + off, *uvh = a.uv + off;
  float qr[CPT], dor[CPT], uqr[CPT];
  load_row<CPT>(qr, a.q + off, row, a.N, a.d, part);
  load_row<CPT>(dor, a.dout + off, row, a.N, a.d, part);
  load_row<CPT>(uqr, a.uq + off, row, a.N, a.d, part);
  const size_t prow = static_cast<size_t>(bh) * a.Np + min(row, a.Np - 1);
  const float L = row < a.N ? a.lse_pad[prow] : INFINITY;
  const float D = row < a.N ? a.d_pad[prow] : 0.f;
  const int last_row = min(a.N - 1, static_cast<int>(blockIdx.x) * R + R - 1);
  const int key_end = a.causal ? last_row + 1 : a.N;

  float x1[CPT], x2[CPT], x3[CPT], x4[CPT], y1[CPT], y2[CPT], y3[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) x1[c] = x2[c] = x3[c] = x4[c] = y1[c] = y2[c] = y3[c] = 0.f;
  float r = 0.f, t1 = 0.f, t3 = 0.f;
  for (int k0 = 0; k0 < key_end; k0 += kRows) {
    __syncthreads();
    stage<DP>(sK, kh, k0, a.N, a.d);
    stage<DP>(sV, vh, k0, a.N, a.d);
    stage<DP>(sUK, ukh, k0, a.N, a.d);
    stage<DP>(sUV, uvh, k0, a.N, a.d);
    __syncthreads();
    for (int u = 0; u < kRows; ++u) {
      const int key = k0 + u;
      const float sc = group_sum<TPR>(dot<DP, CPT>(qr, sK, u, part)) * a.scale;
      const float dp = group_sum<TPR>(dot<DP, CPT>(dor, sV, u, part));
      const float m =
          group_sum<TPR>(dot<DP, CPT>(uqr, sK, u, part) + dot<DP, CPT>(qr, sUK, u, part)) * a.scale;
      const float w = group_sum<TPR>(dot<DP, CPT>(dor, sUV, u, part));
      const bool keep = row < a.N && key < a.N && (!a.causal || key <= row);
      const float p = keep ? expf(sc - L) : 0.f;
      r = fmaf(p, m, r);
      t1 = fmaf(p * m, dp, t1);
      t3 = fmaf(p, w, t3);
      const float a1 = p * (dp - D);
      const float a2 = p * fmaf(m, dp - D, w);
      const float a3 = p * dp;
      const float b1 = p * m;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int ch = CPT * part + c;
        const float kk = sK[u][ch], vv = sV[u][ch];
        x1[c] = fmaf(a1, sUK[u][ch], x1[c]);
        x2[c] = fmaf(a2, kk, x2[c]);
        x3[c] = fmaf(a3, kk, x3[c]);
        x4[c] = fmaf(p, kk, x4[c]);
        y1[c] = fmaf(b1, vv, y1[c]);
        y2[c] = fmaf(p, vv, y2[c]);
        y3[c] = fmaf(p, sUV[u][ch], y3[c]);
      }
    }
  }
  const float g = t1 - 2.f * r * D + t3;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    x1[c] = x1[c] + x2[c] - r * x3[c] - g * x4[c];  // gQ / s
    y1[c] = y1[c] - r * y2[c] + y3[c];              // gdO
  }
  store_row<CPT>(a.gq + off, x1, a.scale, row, a.N, a.d, part);
  store_row<CPT>(a.gdout + off, y1, 1.f, row, a.N, a.d, part);
  if (part == 0 && row < a.Np) {
    a.r_pad[prow] = row < a.N ? r : 0.f;
    a.g_pad[prow] = row < a.N ? g : 0.f;
  }
}

// ------------------------------------------------------------ key rows
template <int DP, int CPT>
__global__ void __launch_bounds__(128) bob_cols_f32_kernel(const BobArgs a) {
  constexpr int TPR = DP / CPT;
  constexpr int R = 128 / TPR;
  __shared__ float sQ[kRows][DP], sdO[kRows][DP], sUQ[kRows][DP];
  __shared__ float sL[kRows], sD[kRows], sR[kRows], sG[kRows];
  const int bh = blockIdx.y;
  const int key = blockIdx.x * R + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const size_t off = static_cast<size_t>(bh) * a.N * a.d;
  const size_t poff = static_cast<size_t>(bh) * a.Np;
  float kr[CPT], vr[CPT], ukr[CPT], uvr[CPT];
  load_row<CPT>(kr, a.k + off, key, a.N, a.d, part);
  load_row<CPT>(vr, a.v + off, key, a.N, a.d, part);
  load_row<CPT>(ukr, a.uk + off, key, a.N, a.d, part);
  load_row<CPT>(uvr, a.uv + off, key, a.N, a.d, part);
  float gk[CPT], gv[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) gk[c] = gv[c] = 0.f;
  const int first_key = blockIdx.x * R;
  const int q_begin = a.causal ? (first_key / kRows) * kRows : 0;
  for (int q0 = q_begin; q0 < a.N; q0 += kRows) {
    __syncthreads();
    stage<DP>(sQ, a.q + off, q0, a.N, a.d);
    stage<DP>(sdO, a.dout + off, q0, a.N, a.d);
    stage<DP>(sUQ, a.uq + off, q0, a.N, a.d);
    if (threadIdx.x < kRows) {
      const int qi = q0 + threadIdx.x;
      const bool in = qi < a.N;
      sL[threadIdx.x] = in ? a.lse_pad[poff + qi] : INFINITY;
      sD[threadIdx.x] = in ? a.d_pad[poff + qi] : 0.f;
      sR[threadIdx.x] = in ? a.r_pad[poff + qi] : 0.f;
      sG[threadIdx.x] = in ? a.g_pad[poff + qi] : 0.f;
    }
    __syncthreads();
    for (int u = 0; u < kRows; ++u) {
      const int qi = q0 + u;
      const float sc = group_sum<TPR>(dot<DP, CPT>(kr, sQ, u, part)) * a.scale;
      const float dp = group_sum<TPR>(dot<DP, CPT>(vr, sdO, u, part));
      const float m =
          group_sum<TPR>(dot<DP, CPT>(kr, sUQ, u, part) + dot<DP, CPT>(ukr, sQ, u, part)) * a.scale;
      const float w = group_sum<TPR>(dot<DP, CPT>(uvr, sdO, u, part));
      const bool keep = qi < a.N && key < a.N && (!a.causal || qi >= key);
      const float p = keep ? expf(sc - sL[u]) : 0.f;
      const float ds = p * (dp - sD[u]);
      const float e = p * (m - sR[u]);
      const float ds2 = p * (m * (dp - sD[u]) - sR[u] * dp + w - sG[u]);
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int ch = CPT * part + c;
        gk[c] = fmaf(ds, sUQ[u][ch], fmaf(ds2, sQ[u][ch], gk[c]));
        gv[c] = fmaf(e, sdO[u][ch], gv[c]);
      }
    }
  }
  store_row<CPT>(a.gk + off, gk, a.scale, key, a.N, a.d, part);
  store_row<CPT>(a.gv + off, gv, 1.f, key, a.N, a.d, part);
}

// The query-row kernel keeps seven accumulators per row, so it always holds
// 8 channels per thread; the key-row kernel takes CPT.
template <int DP, int CPT>
cudaError_t bob_dp(const BobArgs& a, int BH, cudaStream_t s) {
  constexpr int RR = 128 / (DP / 8);
  bob_rows_f32_kernel<DP, 8><<<dim3((a.N + RR - 1) / RR, BH), 128, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr int RC = 128 / (DP / CPT);
  bob_cols_f32_kernel<DP, CPT><<<dim3((a.N + RC - 1) / RC, BH), 128, 0, s>>>(a);
  return cudaGetLastError();
}

// 16 channels per thread while that still gives two CTAs per SM, else 8
template <int DP>
cudaError_t bob_pick(const BobArgs& a, int BH, cudaStream_t s) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int R16 = 128 / (DP / 16);
  const long long ctas16 = static_cast<long long>((a.N + R16 - 1) / R16) * BH;
  if (DP == 128 || ctas16 < 2LL * sms) return bob_dp<DP, 8>(a, BH, s);
  return bob_dp<DP, 16>(a, BH, s);
}

}  // namespace

cudaError_t launch_bob_f32(const float* q, const float* k, const float* v, const float* dout,
                           const float* uq, const float* uk, const float* uv, float* gq,
                           float* gk, float* gv, float* gdout, int BH, int N, int d, bool causal,
                           float scale, const Workspace& ws, float* r_pad, float* g_pad,
                           cudaStream_t s) {
  BobArgs a{q, k, v, dout, uq, uk, uv, gq, gk, gv, gdout, ws.lse_pad, ws.d_pad,
            r_pad, g_pad, N, ws.Np, d, causal ? 1 : 0, scale};
  if (d <= 32) return bob_pick<32>(a, BH, s);
  if (d <= 64) return bob_pick<64>(a, BH, s);
  return bob_pick<128>(a, BH, s);
}

}  // namespace csa
