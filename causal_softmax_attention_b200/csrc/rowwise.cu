// Row-wise, memory-bound stages of the backward.
//
// preprocess: D_i = sum_c dO_ic O_ic for every row (the "sums weighted by the
//   softmax" of ddx issue #243 item 2, which equal sum_j P_ij dP_ij), a copy
//   of LSE padded to whole 128-row tiles (for the bf16 path as -LSE*log2(e),
//   the term the tensor-core backward adds to its scaled scores, -inf past N;
//   for the f32 path LSE itself, +inf past N: either way padded query rows get
//   P = 0), the zeroed fp32 dQ accumulator (bf16 path) and the zeroed status
//   word.
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
      lse_pad[r] = l == -INFINITY ? -INFINITY : -(l * kLog2e);
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
// 4*c4 + e). One CTA per half tile (64 rows): the rows' accumulator columns
// are read as 16-byte vectors in storage order (each column group of the 64
// rows is 1 KB of contiguous memory), transposed through shared memory, and
// written as bf16 rows, consecutive threads covering consecutive 8-byte
// pieces of a row. Both sides of HBM traffic are therefore fully coalesced,
// and every index is 32-bit arithmetic on the CTA's own tile.
constexpr int kConvRows = 64;

template <int D>
__global__ void __launch_bounds__(256)
    dq_convert_kernel(const float4* __restrict__ acc, __nv_bfloat16* __restrict__ dq, int N, int T,
                      float scale, RowStrides qs) {
  constexpr int C4 = D / 4;       // 16-byte column groups per row
  constexpr int LD = C4 + 1;      // padded row length in shared memory (float4)
  __shared__ float4 tile[kConvRows * LD];
  const int half = blockIdx.x & 1;
  const int t = (blockIdx.x >> 1) % T;
  const int bh = (blockIdx.x >> 1) / T;
  const int r0 = half * kConvRows;
  const float4* src = acc + (static_cast<size_t>(bh) * T + t) * (C4 * kTile);
#pragma unroll
  for (int f = threadIdx.x; f < C4 * kConvRows; f += 256) {
    const int c4 = f / kConvRows, r = f % kConvRows;
    tile[r * LD + c4] = src[c4 * kTile + r0 + r];
  }
  __syncthreads();
  const int row0 = t * kTile + r0;
  __nv_bfloat16* base = dq + qs.head(bh);
#pragma unroll
  for (int f = threadIdx.x; f < C4 * kConvRows; f += 256) {
    const int r = f / C4, c4 = f % C4;
    if (row0 + r >= N) continue;
    const float4 x = tile[r * LD + c4];
    __nv_bfloat162 h[2];
    h[0] = __floats2bfloat162_rn(x.x * scale, x.y * scale);
    h[1] = __floats2bfloat162_rn(x.z * scale, x.w * scale);
    *reinterpret_cast<uint2*>(base + static_cast<long long>(row0 + r) * qs.sn + 4 * c4) =
        *reinterpret_cast<const uint2*>(h);
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
  // (a workspace without a dQ accumulator -- the backward-over-backward's --
  // skips the zeroing)
  const size_t acc_vecs = ws.dq_acc != nullptr ? rows * d / 4 : 0;
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
  const unsigned grid = static_cast<unsigned>(BH) * static_cast<unsigned>(T) * (kTile / kConvRows);
  const float4* acc = reinterpret_cast<const float4*>(ws.dq_acc);
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(dq);
  switch (d) {
    case 32: dq_convert_kernel<32><<<grid, 256, 0, s>>>(acc, out, N, T, scale, qs); break;
    case 64: dq_convert_kernel<64><<<grid, 256, 0, s>>>(acc, out, N, T, scale, qs); break;
    case 128: dq_convert_kernel<128><<<grid, 256, 0, s>>>(acc, out, N, T, scale, qs); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace csa
