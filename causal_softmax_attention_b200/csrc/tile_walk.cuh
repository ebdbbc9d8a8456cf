// Block-mask walks in shared memory: one CTA's line of a [T][T] block mask
// (a key tile's column in the backward, a query tile's row in the forward)
// turned into two bitmaps once, so that every role finds its next tile with
// a shared-memory word scan instead of byte loads from global memory.
//
// Tile kinds (one byte per 128 x 128 tile): 0 the tile takes no part, 2 the
// causal filter inside the tile, any other value the whole tile. Bit t of
// `act` is set for a tile that takes part, bit t of `kind2` for kind 2.
#pragma once

#include <cstddef>
#include <cstdint>

namespace csa {

// All THREADS threads of the block call this with the same arguments. Reads
// line[t * stride] for t < T; writes ceil(T / 32) words of each bitmap
// (rounded up to whole rounds of THREADS tiles: the caller provides
// round_up(T, THREADS) / 32 words). Bits past T are 0. The caller
// synchronises the block before the bitmaps are read.
template <int THREADS>
__device__ __forceinline__ void build_tile_bits(const uint8_t* line, size_t stride, int T,
                                                uint32_t* act, uint32_t* kind2) {
  static_assert(THREADS % 32 == 0, "whole warps");
  constexpr int kBatch = 4;  // rounds whose loads are in flight together
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int t0 = 0; t0 < T; t0 += kBatch * THREADS) {
    uint8_t v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int t = t0 + b * THREADS + static_cast<int>(threadIdx.x);
      v[b] = t < T ? line[static_cast<size_t>(t) * stride] : 0;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int w0 = (t0 + b * THREADS) >> 5;  // first word of this round
      if (t0 + b * THREADS >= T) break;        // uniform: every thread sees the same t0
      const uint32_t a = __ballot_sync(0xffffffffu, v[b] != 0);
      const uint32_t k = __ballot_sync(0xffffffffu, v[b] == 2);
      if (lane == 0) {
        act[w0 + warp] = a;
        kind2[w0 + warp] = k;
      }
    }
  }
}

// First set bit after position i (i >= -1), or T if none.
__device__ __forceinline__ int next_set_bit(const uint32_t* act, int T, int i) {
  int t = i + 1;
  while (t < T) {
    const uint32_t w = act[t >> 5] >> (t & 31);
    if (w != 0u) return t + __ffs(static_cast<int>(w)) - 1;
    t = (t | 31) + 1;
  }
  return T;
}

__device__ __forceinline__ bool bit_set(const uint32_t* bits, int t) {
  return (bits[t >> 5] >> (t & 31)) & 1u;
}

}  // namespace csa
