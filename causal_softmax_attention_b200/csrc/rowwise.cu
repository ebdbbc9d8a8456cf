// Row-wise, memory-bound stages of the backward.
//
// preprocess: D_i = sum_c dO_ic O_ic for every row (the "sums weighted by the
//   softmax" of ddx issue #243 item 2, which equal sum_j P_ij dP_ij), a copy
//   of LSE padded to whole 128-row tiles (scaled by log2(e) for the bf16 path,
//   +inf past N so padded query rows get P = 0), the zeroed fp32 dQ
//   accumulator (bf16 path) and the zeroed status word.
// dq_convert: dQ = scale * accumulator, rounded to bf16.
//
// Both are bound by HBM bandwidth: 16-byte vector loads/stores, one thread
// group per row, grid-stride loops sized to the SM count.
#include <cuda_bf16.h>

#include "common.cuh"

namespace csa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// bf16 rows: G = d/8 lanes per row, one 16-byte vector (8 channels) each.
template <int G>
__global__ void __launch_bounds__(256)
    preprocess_bf16_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dout,
                           const float* __restrict__ lse, float* __restrict__ lse_pad,
                           float* __restrict__ d_pad, float4* __restrict__ dq_acc,
                           size_t acc_vecs, int* status, int BH, int N, int Np,
                           RowStrides os) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = kStatusOk;
  const size_t total_rows = static_cast<size_t>(BH) * Np;
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t nthreads = static_cast<size_t>(gridDim.x) * blockDim.x;
  const int lane = threadIdx.x & 31;
  const int sub = lane % G;
  constexpr int kRowsPerWarp = 32 / G;
  // Loop bounds are uniform across the warp so every lane reaches the shuffles.
  for (size_t r0 = tid / 32 * kRowsPerWarp; r0 < total_rows; r0 += nthreads / 32 * kRowsPerWarp) {
    const size_t r = r0 + lane / G;
    const bool active = r < total_rows;
    const int bh = static_cast<int>(r / Np);
    const int i = static_cast<int>(r % Np);
    float acc = 0.f;
    if (active && i < N) {
      const size_t idx = static_cast<size_t>(os.row(bh, i) / 8) + sub;  // 16-byte vectors
      const uint4 a = o[idx], b = dout[idx];
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(pa[e]);
        const float2 fb = __bfloat1622float2(pb[e]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int off = 1; off < G; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (active && sub == 0) {
      d_pad[r] = acc;
      // a row with no kept key (LSE = -inf) must give P = 0, like a padded row
      const float l = i < N ? lse[static_cast<size_t>(bh) * N + i] : INFINITY;
      lse_pad[r] = l == -INFINITY ? INFINITY : l * kLog2e;
    }
  }
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (size_t v = tid; v < acc_vecs; v += nthreads) dq_acc[v] = zero;
}

// fp32 rows of any width: one warp per row.
__global__ void __launch_bounds__(256)
    preprocess_f32_kernel(const float* __restrict__ o, const float* __restrict__ dout,
                          const float* __restrict__ lse, float* __restrict__ lse_pad,
                          float* __restrict__ d_pad, int* status, int BH, int N, int Np, int d,
                          RowStrides os) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = kStatusOk;
  const size_t total_rows = static_cast<size_t>(BH) * Np;
  const size_t warp0 = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const size_t nwarps = static_cast<size_t>(gridDim.x) * blockDim.x / 32;
  const int lane = threadIdx.x & 31;
  for (size_t r = warp0; r < total_rows; r += nwarps) {
    const int bh = static_cast<int>(r / Np);
    const int i = static_cast<int>(r % Np);
    float acc = 0.f;
    if (i < N) {
      const size_t row = static_cast<size_t>(os.row(bh, i));
      for (int c = lane; c < d; c += 32) acc = fmaf(o[row + c], dout[row + c], acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      d_pad[r] = acc;
      const float l = i < N ? lse[static_cast<size_t>(bh) * N + i] : INFINITY;
      lse_pad[r] = l == -INFINITY ? INFINITY : l;
    }
  }
}

// Accumulator layout [BH][T][d/4][128][4]: element (row r of tile t, column
// 4*c4 + e). Each thread converts 8 consecutive columns of one row.
__global__ void __launch_bounds__(256)
    dq_convert_kernel(const float4* __restrict__ acc, __nv_bfloat16* __restrict__ dq, int BH,
                      int N, int T, int d, float scale, RowStrides qs) {
  const int g8 = d / 8;
  const size_t total = static_cast<size_t>(BH) * T * g8 * kTile;
  const size_t nthreads = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t id = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; id < total;
       id += nthreads) {
    const int r = static_cast<int>(id % kTile);
    size_t rest = id / kTile;
    const int g = static_cast<int>(rest % g8);
    rest /= g8;
    const int tile = static_cast<int>(rest % T);
    const int bh = static_cast<int>(rest / T);
    const int i = tile * kTile + r;
    if (i >= N) continue;
    const size_t a0 = ((static_cast<size_t>(bh) * T + tile) * (d / 4) + 2 * g) * kTile + r;
    const float4 x = acc[a0];
    const float4 y = acc[a0 + kTile];
    __nv_bfloat162 h[4];
    h[0] = __floats2bfloat162_rn(x.x * scale, x.y * scale);
    h[1] = __floats2bfloat162_rn(x.z * scale, x.w * scale);
    h[2] = __floats2bfloat162_rn(y.x * scale, y.y * scale);
    h[3] = __floats2bfloat162_rn(y.z * scale, y.w * scale);
    *reinterpret_cast<uint4*>(dq + qs.row(bh, i) + 8 * g) =
        *reinterpret_cast<const uint4*>(h);
  }
}

int sm_count() {
  static int cached = 0;
  if (cached == 0) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached = n > 0 ? n : 148;
  }
  return cached;
}

unsigned grid_for(size_t threads_needed) {
  const size_t per_wave = static_cast<size_t>(sm_count()) * 8;  // 8 x 256-thread blocks per SM
  size_t blocks = (threads_needed + 255) / 256;
  if (blocks > per_wave) blocks = per_wave;
  return static_cast<unsigned>(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_preprocess(const void* o, const void* dout, const float* lse, int BH, int N,
                              int d, bool bf16, const RowStrides& os, const Workspace& ws,
                              cudaStream_t s) {
  const size_t rows = static_cast<size_t>(BH) * ws.Np;
  if (!bf16) {
    preprocess_f32_kernel<<<grid_for(rows * 32), 256, 0, s>>>(
        static_cast<const float*>(o), static_cast<const float*>(dout), lse, ws.lse_pad,
        ws.d_pad, ws.status, BH, N, ws.Np, d, os);
    return cudaGetLastError();
  }
  const size_t acc_vecs = rows * d / 4;
  const int G = d / 8;
  const unsigned grid = grid_for(rows * G > acc_vecs ? rows * G : acc_vecs);
  const uint4* po = static_cast<const uint4*>(o);
  const uint4* pd = static_cast<const uint4*>(dout);
  float4* acc = reinterpret_cast<float4*>(ws.dq_acc);
  switch (G) {
    case 4:
      preprocess_bf16_kernel<4><<<grid, 256, 0, s>>>(po, pd, lse, ws.lse_pad, ws.d_pad, acc,
                                                     acc_vecs, ws.status, BH, N, ws.Np, os);
      break;
    case 8:
      preprocess_bf16_kernel<8><<<grid, 256, 0, s>>>(po, pd, lse, ws.lse_pad, ws.d_pad, acc,
                                                     acc_vecs, ws.status, BH, N, ws.Np, os);
      break;
    case 16:
      preprocess_bf16_kernel<16><<<grid, 256, 0, s>>>(po, pd, lse, ws.lse_pad, ws.d_pad, acc,
                                                      acc_vecs, ws.status, BH, N, ws.Np, os);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_dq_convert(void* dq, int BH, int N, int d, float scale, const RowStrides& qs,
                              const Workspace& ws, cudaStream_t s) {
  const int T = ws.Np / kTile;
  const size_t total = static_cast<size_t>(BH) * T * (d / 8) * kTile;
  dq_convert_kernel<<<grid_for(total), 256, 0, s>>>(reinterpret_cast<const float4*>(ws.dq_acc),
                                                    static_cast<__nv_bfloat16*>(dq), BH, N, T, d,
                                                    scale, qs);
  return cudaGetLastError();
}

}  // namespace csa
