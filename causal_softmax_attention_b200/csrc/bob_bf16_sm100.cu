// Backward-over-backward of causal softmax attention on the sm_100a tensor
// cores (tcgen05): bf16 inputs and outputs, fp32 accumulation in tensor
// memory. The gradient, with respect to Q, K, V and dO, of
//   L2 = <U_Q, dQ> + <U_K, dK> + <U_V, dV>,
// where (dQ, dK, dV) is attention's first backward -- the operation of the
// FlashBoB listing ("Approaching I/O-optimality for Approximate Attention",
// abstract): exact differentiation through the backward pass, in passes over
// the scores that first form two row-wise scalars. Per score pair (i, j),
// recomputed from the rows alone (s the scale, D_i = sum_c dO_ic O_ic):
//
//   P = exp(s q_i.k_j - LSE_i)      dP = dO_i.v_j
//   M = s (u_Q,i.k_j + q_i.u_K,j)   W  = dO_i.u_V,j
//   r_i = sum_j P M                 g_i = sum_j P (M dP + W) - 2 r_i D_i
//   dS = P (dP - D_i)   E = P (M - r_i)   dS2 = P (M (dP - D_i) - r_i dP + W - g_i)
//
//   gQ_i = s sum_j (dS u_K,j + dS2 k_j)     gdO_i = sum_j (E v_j + P u_V,j)
//   gK_j = s sum_i (dS u_Q,i + dS2 q_i)     gV_j  = sum_i E dO_i
//
// (g uses sum_j P dP = D_i.) Every sum over j or i is a dense contraction of a
// 128 x 64 tile, so all of them run as tcgen05 MMAs:
//
//   rows kernel (one CTA per query tile, lanes = queries): key tiles in 64-key
//     halves; S, dP, M (two MMAs into one accumulator) and W by SS MMAs into
//     four 64-column TMEM blocks. A first sweep over the key tiles forms the
//     row sums r and g in registers (and stores them for the columns kernel);
//     a second sweep writes dS, dS2, E and P as bf16 over the blocks they came
//     from and accumulates gQ / s += dS U_K + dS2 K and gdO += E V + P U_V with
//     TS MMAs (A from tensor memory, B the key tiles read MN-major).
//   columns kernel (one CTA per key tile, lanes = keys): query tiles in
//     64-query halves; S^T, dP^T, M^T, W^T, then dS^T, dS2^T, E^T from the
//     stored r, g and gK / s += dS^T U_Q + dS2^T Q, gV += E^T dO.
//
// Warps (384 threads): 0-7 two element-wise warpgroups (thread t of group g
// owns TMEM lane t and the columns [32g, 32g+32) of each 64-column block);
// warp 8 issues the MMAs, warp 9 the TMA loads; 10-11 idle. Each half runs
// score MMAs -> element-wise pass -> accumulating MMAs in turn; every wait is
// bounded and reports a timeout. Nothing N x N is stored.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace {

using namespace sm100;

constexpr int kBobThreads = 384;
constexpr int kBobEThreads = 256;
constexpr int kBobMmaWarp = 8;
constexpr int kBobTmaWarp = 9;

template <int D>
struct BobLayout {
  static constexpr int CH = D >= 64 ? 64 : D;   // TMA box width (elements)
  static constexpr int NCH = D / CH;
  static constexpr int ROWB = CH * 2;
  static constexpr int CHUNK = kTile * ROWB;    // one [128][CH] box
  static constexpr int TILE = NCH * CHUNK;      // one [128][D] bf16 tile
  static constexpr uint32_t SWZ = ROWB == 128 ? kSwizzle128B : kSwizzle64B;
  // seven tiles: the rows kernel keeps Q, dO, U_Q and streams K, V, U_K,
  // U_V; the columns kernel keeps K, V, U_K, U_V and streams Q, dO, U_Q
  static constexpr int VEC_OFF = 7 * TILE;      // columns: [4][128] f32 per-query terms;
                                                // rows: [2][2][128] f32 row-sum exchange
  static constexpr int BAR_OFF = VEC_OFF + 4 * 512;
  static constexpr int MISC_OFF = BAR_OFF + 16 * 8;
  static constexpr int BYTES = MISC_OFF + 64;
  // d = 128 fills the window exactly (its base must then be 1024-byte
  // aligned, checked at run time); smaller d keep 1 KB of alignment slack
  // and at least ~118 KB, so that one CTA owns an SM's tensor memory
  static constexpr bool EXACT = D == 128;
  static constexpr int ALLOC =
      EXACT ? BYTES : ((BYTES + 1024) > 118 * 1024 ? BYTES + 1024 : 118 * 1024);
  // TMEM: S, dP, M, W of one 64-wide half, then two fp32 accumulators
  static constexpr uint32_t T_S = 0, T_DP = 64, T_M = 128, T_W = 192;
  static constexpr uint32_t T_A0 = 256, T_A1 = 256 + D;
  static constexpr uint32_t T_COLS = 512;
  static_assert(T_A1 + D <= T_COLS, "TMEM columns exceeded");
};

enum BobBar {
  O_RES = 0, O_FULL, O_EMPTY, O_SFULL, O_EDONE, O_ACC, O_DONE, O_XCH, O_FINAL, O_COUNT
};
static_assert(O_COUNT <= 16, "barrier slots");

struct BobParams {
  const float* nlse;  // [BH][Np]: -LSE * log2(e), -inf past N
  const float* dvec;  // [BH][Np]: D, 0 past N
  float* r_pad;       // [BH][Np]: row scalar r (written by the rows kernel)
  float* g_pad;       // [BH][Np]: row scalar g
  __nv_bfloat16* out0;  // rows kernel: gQ; columns kernel: gK   ([BH][N][D])
  __nv_bfloat16* out1;  // rows kernel: gdO; columns kernel: gV
  int* status;
  int N, Np, T, BH, H, G, causal;  // H splits bh into the tensor maps' (head, batch)
  float scale, scale_log2;
  uint64_t wait_cycles;
};

template <int D>
__device__ __forceinline__ uint64_t bdesc_kmajor(uint32_t tile, int kk) {
  using L = BobLayout<D>;
  const int e = kk * 16;
  return smem_desc(tile + (e / L::CH) * L::CHUNK + (e % L::CH) * 2, 16, 8 * L::ROWB, L::SWZ);
}
template <int D>
__device__ __forceinline__ uint64_t bdesc_mnmajor(uint32_t tile, int kk) {
  using L = BobLayout<D>;
  return smem_desc(tile + kk * 16 * L::ROWB, L::CHUNK, 8 * L::ROWB, L::SWZ);
}
// TMEM column of the bf16 pair holding element k (k even) of a 64-wide half:
// each element-wise group packs its 32 elements into the first 16 of its own
// 32 columns.
__host__ __device__ constexpr uint32_t h_col(int k) { return 32 * (k >> 5) + ((k & 31) >> 1); }

// Score MMAs of one 64-wide half: four [128 x 64] fp32 blocks
//   T_S  = A0 B0^T,  T_DP = A1 B1^T,  T_M = A2 B2^T + A3 B3^T,  T_W = A4 B4^T
// with the A tiles [128][D] and the B tiles' 64 rows starting at `boff`.
template <int D>
__device__ __forceinline__ void issue_scores(uint32_t tmem, uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t a4, uint32_t b0, uint32_t b1,
                                             uint32_t b2, uint32_t b3, uint32_t b4,
                                             uint32_t boff) {
  using L = BobLayout<D>;
  constexpr uint32_t ID = idesc_bf16(128, 64, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    mma_ss(tmem + L::T_S, bdesc_kmajor<D>(a0, kk), bdesc_kmajor<D>(b0 + boff, kk), ID, kk > 0);
    mma_ss(tmem + L::T_DP, bdesc_kmajor<D>(a1, kk), bdesc_kmajor<D>(b1 + boff, kk), ID, kk > 0);
    mma_ss(tmem + L::T_M, bdesc_kmajor<D>(a2, kk), bdesc_kmajor<D>(b2 + boff, kk), ID, kk > 0);
    mma_ss(tmem + L::T_W, bdesc_kmajor<D>(a4, kk), bdesc_kmajor<D>(b4 + boff, kk), ID, kk > 0);
  }
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_ss(tmem + L::T_M, bdesc_kmajor<D>(a3, kk), bdesc_kmajor<D>(b3 + boff, kk), ID, 1);
}

// acc (+)= [packed bf16 block at `blk`] x B, B the 64 rows of a tile starting
// at row 64 h, read MN-major (K = those 64 rows, N = D channels).
template <int D>
__device__ __forceinline__ void issue_acc(uint32_t tmem, uint32_t acc, uint32_t blk, uint32_t b,
                                          int h, bool accumulate) {
  constexpr uint32_t ID = idesc_bf16(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_ts(tmem + acc, tmem + blk + h_col(16 * kk), bdesc_mnmajor<D>(b, 4 * h + kk), ID,
           (accumulate || kk > 0) ? 1u : 0u);
}

// Epilogue: 128 lanes x D fp32 columns of `acc` -> bf16 rows (x mul); group g
// writes channels [g D/2, (g+1) D/2); rows at or past N are not written.
template <int D>
__device__ __forceinline__ void store_acc(uint32_t lane_base, uint32_t acc, __nv_bfloat16* row,
                                          bool row_ok, int g, float mul) {
  constexpr int HALF = D / 2;
  constexpr int W = HALF >= 32 ? 32 : HALF;
#pragma unroll 1
  for (int c = 0; c < HALF; c += W) {
    uint32_t v[W];
    tmem_ld<W>(lane_base + acc + g * HALF + c, v);
    tmem_ld_wait(v);
    if (row_ok) {
#pragma unroll
      for (int u = 0; u < W; u += 8) {
        uint4 o;
        o.x = pack_bf16x2(mul * __uint_as_float(v[u + 0]), mul * __uint_as_float(v[u + 1]));
        o.y = pack_bf16x2(mul * __uint_as_float(v[u + 2]), mul * __uint_as_float(v[u + 3]));
        o.z = pack_bf16x2(mul * __uint_as_float(v[u + 4]), mul * __uint_as_float(v[u + 5]));
        o.w = pack_bf16x2(mul * __uint_as_float(v[u + 6]), mul * __uint_as_float(v[u + 7]));
        *reinterpret_cast<uint4*>(row + g * HALF + c + u) = o;
      }
    }
  }
}

// Common CTA prologue: 1024-byte aligned window, barriers, TMEM.
template <int D>
__device__ __forceinline__ bool bob_setup(uint8_t* smem_raw, uint8_t*& smem, uint64_t*& bars,
                                          uint32_t& tmem, volatile int*& abort_flag,
                                          const volatile int*& never, int* status) {
  using L = BobLayout<D>;
  smem = L::EXACT ? smem_raw
                  : reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(status, -3);
    return false;
  }
  bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  never = reinterpret_cast<const volatile int*>(smem + L::MISC_OFF + 8);
  if (threadIdx.x == 0) {
    mbar_init(&bars[O_RES], 1);
    mbar_init(&bars[O_FULL], 1);
    mbar_init(&bars[O_EMPTY], 1);
    mbar_init(&bars[O_SFULL], 1);
    mbar_init(&bars[O_EDONE], kBobEThreads);
    mbar_init(&bars[O_ACC], 1);
    mbar_init(&bars[O_DONE], 1);
    mbar_init(&bars[O_XCH], kBobEThreads);
    mbar_init(&bars[O_FINAL], 1);
    *abort_flag = 0;
    *const_cast<volatile int*>(never) = 0;
    fence_barrier_init();
  }
  if ((threadIdx.x >> 5) == 0) {
    tmem_alloc(tmem_slot, L::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tmem = *tmem_slot;
  return true;
}

template <int D>
__device__ __forceinline__ void bob_teardown(uint32_t tmem) {
  using L = BobLayout<D>;
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::T_COLS);
  }
}

// ============================================================== rows kernel
// Tiles: 0 Q_i, 1 dO_i, 2 U_Q,i (resident); 3 K_j, 4 V_j, 5 U_K,j, 6 U_V,j.
template <int D>
__global__ void __launch_bounds__(kBobThreads, 1)
    bob_rows_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_uq,
                         const __grid_constant__ CUtensorMap tm_uk,
                         const __grid_constant__ CUtensorMap tm_uv, const BobParams p) {
  using L = BobLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem;
  uint64_t* bars;
  uint32_t tmem;
  volatile int* abort_flag;
  const volatile int* never;
  if (!bob_setup<D>(smem_raw, smem, bars, tmem, abort_flag, never, p.status)) return;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  // CTA order: heads in groups of G (their key tiles stay in L2 while the
  // group's query tiles pass), longest query tile first inside a group
  const int per_group = p.T * p.G;
  const int g0 = (blockIdx.x / per_group) * p.G;
  const int rr = blockIdx.x % per_group;
  const int gs = min(p.G, p.BH - g0);
  const int it_q = p.causal ? p.T - 1 - rr / gs : rr / gs;
  const int bh = g0 + rr % gs;
  const int hh = bh % p.H, hb = bh / p.H;  // TMA coordinates
  const int i0 = it_q * kTile;
  const int n_kt = p.causal ? it_q + 1 : p.T;  // key tiles this query tile meets
  const int n_loads = 2 * n_kt;                 // two sweeps
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, kStatusTimeout);
  };

  if (warp == kBobTmaWarp) {
    // ------------------------------------------------ TMA producer
    if (elect_one_sync()) {
      for (const CUtensorMap* m : {&tm_q, &tm_k, &tm_v, &tm_do, &tm_uq, &tm_uk, &tm_uv})
        prefetch_tensormap(m);
      mbar_arrive_expect_tx(&bars[O_RES], 3 * L::TILE);
      for (int c = 0; c < L::NCH; ++c) {
        tma_load_4d(smem + 0 * L::TILE + c * L::CHUNK, &tm_q, &bars[O_RES], c * L::CH, i0, hh, hb);
        tma_load_4d(smem + 1 * L::TILE + c * L::CHUNK, &tm_do, &bars[O_RES], c * L::CH, i0, hh, hb);
        tma_load_4d(smem + 2 * L::TILE + c * L::CHUNK, &tm_uq, &bars[O_RES], c * L::CH, i0, hh, hb);
      }
      bool ok = true;
      int issued = 0;
      for (int n = 0; n < n_loads; ++n) {
        const int j0 = (n % n_kt) * kTile;
        if (n > 0 && !(ok = mbar_wait(&bars[O_EMPTY], (n - 1) & 1, p.wait_cycles, abort_flag)))
          break;
        mbar_arrive_expect_tx(&bars[O_FULL], 4 * L::TILE);
        for (int c = 0; c < L::NCH; ++c) {
          tma_load_4d(smem + 3 * L::TILE + c * L::CHUNK, &tm_k, &bars[O_FULL], c * L::CH, j0, hh, hb);
          tma_load_4d(smem + 4 * L::TILE + c * L::CHUNK, &tm_v, &bars[O_FULL], c * L::CH, j0, hh, hb);
          tma_load_4d(smem + 5 * L::TILE + c * L::CHUNK, &tm_uk, &bars[O_FULL], c * L::CH, j0, hh, hb);
          tma_load_4d(smem + 6 * L::TILE + c * L::CHUNK, &tm_uv, &bars[O_FULL], c * L::CH, j0, hh, hb);
        }
        ++issued;
      }
      if (!ok) fail();
      // every load issued has landed before the CTA can exit (bounded; one
      // buffer, so only the last can still be in flight)
      mbar_wait(&bars[O_RES], 0, p.wait_cycles, never);
      if (issued > 0) mbar_wait(&bars[O_FULL], (issued - 1) & 1, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp == kBobMmaWarp) {
    // ------------------------------------------------ MMA issuer
    if (elect_one_sync()) {
      const uint32_t sQ = sbase, sDO = sbase + L::TILE, sUQ = sbase + 2 * L::TILE;
      const uint32_t sK = sbase + 3 * L::TILE, sV = sbase + 4 * L::TILE;
      const uint32_t sUK = sbase + 5 * L::TILE, sUV = sbase + 6 * L::TILE;
      auto wait = [&](int b, uint32_t parity) {
        return mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag);
      };
      bool ok = wait(O_RES, 0);
      int hn = 0, acc_n = 0;
      for (int n = 0; ok && n < n_loads; ++n) {
        const bool second = n >= n_kt;
        if (!(ok = wait(O_FULL, n & 1))) break;
        tc_fence_after();
        for (int h = 0; h < 2; ++h, ++hn) {
          // S = Q K_h^T, dP = dO V_h^T, M = U_Q K_h^T + Q U_K,h^T, W = dO U_V,h^T
          issue_scores<D>(tmem, sQ, sDO, sUQ, sQ, sDO, sK, sV, sK, sUK, sUV,
                          static_cast<uint32_t>(64 * h * L::ROWB));
          mma_commit(&bars[O_SFULL]);
          if (!(ok = wait(O_EDONE, hn & 1))) break;
          tc_fence_after();
          if (second) {
            // gQ/s += dS U_K,h + dS2 K_h;  gdO += E V_h + P U_V,h
            const bool acc = acc_n > 0;
            issue_acc<D>(tmem, L::T_A0, L::T_S, sUK, h, acc);
            issue_acc<D>(tmem, L::T_A0, L::T_DP, sK, h, true);
            issue_acc<D>(tmem, L::T_A1, L::T_M, sV, h, acc);
            issue_acc<D>(tmem, L::T_A1, L::T_W, sUV, h, true);
            mma_commit(&bars[O_ACC]);
            // the next half's scores overwrite the blocks these MMAs read
            if (!(ok = wait(O_ACC, acc_n & 1))) break;
            tc_fence_after();
            ++acc_n;
          }
        }
        if (!ok) break;
        mma_commit(&bars[O_EMPTY]);  // the key tiles are free once these MMAs complete
      }
      if (ok) {
        mma_commit(&bars[O_DONE]);
      } else {
        fail();
      }
      mma_commit(&bars[O_FINAL]);
      mbar_wait(&bars[O_FINAL], 0, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------ element-wise warpgroups
    const int t = threadIdx.x & 127;  // TMEM lane: query row i0 + t
    const int g = threadIdx.x >> 7;   // columns [32g, 32g+32) of each block
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int row = i0 + t;
    const size_t vrow = static_cast<size_t>(bh) * p.Np + row;
    const float nl = p.nlse[vrow];
    const float dv = p.dvec[vrow];
    float* xch = reinterpret_cast<float*>(smem + L::VEC_OFF);  // [2 sums][2 groups][128]
    auto wait_w = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag));
    };
    float r_sum = 0.f, g_sum = 0.f;  // this group's partial row sums (first sweep)
    float rr_ = 0.f, gg_ = 0.f;      // the row scalars (second sweep)
    bool ok = true;
    int hn = 0;
    for (int n = 0; ok && n < n_loads; ++n) {
      const bool second = n >= n_kt;
      if (n == n_kt) {
        // both groups' partial sums -> r, g of the row (a bounded barrier
        // wait, so that a timed-out group cannot hold the other forever)
        xch[(0 * 2 + g) * 128 + t] = r_sum;
        xch[(1 * 2 + g) * 128 + t] = g_sum;
        mbar_arrive(&bars[O_XCH]);
        if (!(ok = wait_w(O_XCH, 0))) break;
        rr_ = r_sum + xch[(0 * 2 + (g ^ 1)) * 128 + t];
        gg_ = g_sum + xch[(1 * 2 + (g ^ 1)) * 128 + t] - 2.f * rr_ * dv;
        if (g == 0 && CSA_IN_BOUNDS(row < p.Np && bh < p.BH, p.status)) {
          p.r_pad[vrow] = rr_;
          p.g_pad[vrow] = gg_;
        }
      }
      const int j0 = (n % n_kt) * kTile;
      for (int h = 0; h < 2; ++h, ++hn) {
        if (!(ok = wait_w(O_SFULL, hn & 1))) break;
        tc_fence_after();
        const int kb = j0 + 64 * h + 32 * g;  // first key of this thread's 32 columns
        int lim = p.N - kb;                    // columns u >= lim are masked
        if (p.causal && row - kb + 1 < lim) lim = row - kb + 1;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          const uint32_t col = 32 * g + 16 * c;
          uint32_t s[16], dp[16], m[16], w[16];
          tmem_ld16(lane_base + L::T_S + col, s);
          tmem_ld16(lane_base + L::T_DP + col, dp);
          tmem_ld16(lane_base + L::T_M + col, m);
          tmem_ld16(lane_base + L::T_W + col, w);
          tmem_ld_wait(s, dp);
          tmem_ld_wait(m, w);
          uint32_t o_ds[8], o_ds2[8], o_e[8], o_p[8];
#pragma unroll
          for (int u = 0; u < 16; u += 2) {
            float pv[2], ds[2], ds2[2], ev[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int uu = 16 * c + u + e;
              float pp = ex2_approx(fmaf(__uint_as_float(s[u + e]), p.scale_log2, nl));
              if (uu >= lim) pp = 0.f;
              const float mm = p.scale * __uint_as_float(m[u + e]);
              const float dpv = __uint_as_float(dp[u + e]);
              const float wv = __uint_as_float(w[u + e]);
              if (!second) {
                r_sum = fmaf(pp, mm, r_sum);
                g_sum = fmaf(pp, fmaf(mm, dpv, wv), g_sum);
              } else {
                const float x = dpv - dv;
                pv[e] = pp;
                ds[e] = pp * x;
                ds2[e] = pp * (fmaf(mm, x, fmaf(-rr_, dpv, wv)) - gg_);
                ev[e] = pp * (mm - rr_);
              }
            }
            if (second) {
              o_ds[u / 2] = pack_bf16x2(ds[0], ds[1]);
              o_ds2[u / 2] = pack_bf16x2(ds2[0], ds2[1]);
              o_e[u / 2] = pack_bf16x2(ev[0], ev[1]);
              o_p[u / 2] = pack_bf16x2(pv[0], pv[1]);
            }
          }
          if (second) {
            // the packed pairs land in the first 16 of this group's 32
            // columns of each block: chunk c's 8 columns were read above
            const uint32_t oc = 32 * g + 8 * c;
            tmem_st8(lane_base + L::T_S + oc, o_ds);
            tmem_st8(lane_base + L::T_DP + oc, o_ds2);
            tmem_st8(lane_base + L::T_M + oc, o_e);
            tmem_st8(lane_base + L::T_W + oc, o_p);
          }
        }
        if (second) tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[O_EDONE]);
      }
    }
    if (ok) ok = wait_w(O_DONE, 0);
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      const bool row_ok = row < p.N && CSA_IN_BOUNDS(bh < p.BH && it_q < p.T, p.status);
      const size_t orow = (static_cast<size_t>(bh) * p.N + (row_ok ? row : 0)) * D;
      store_acc<D>(lane_base, L::T_A0, p.out0 + orow, row_ok, g, p.scale);
      store_acc<D>(lane_base, L::T_A1, p.out1 + orow, row_ok, g, 1.f);
    }
  }
  bob_teardown<D>(tmem);
}

// ============================================================== columns kernel
// Tiles: 0 K_j, 1 V_j, 2 U_K,j, 3 U_V,j (resident); 4 Q_i, 5 dO_i, 6 U_Q,i.
template <int D>
__global__ void __launch_bounds__(kBobThreads, 1)
    bob_cols_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_uq,
                         const __grid_constant__ CUtensorMap tm_uk,
                         const __grid_constant__ CUtensorMap tm_uv, const BobParams p) {
  using L = BobLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem;
  uint64_t* bars;
  uint32_t tmem;
  volatile int* abort_flag;
  const volatile int* never;
  if (!bob_setup<D>(smem_raw, smem, bars, tmem, abort_flag, never, p.status)) return;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  // CTA order: heads in groups of G, longest key tile (key tile 0) first
  const int per_group = p.T * p.G;
  const int g0 = (blockIdx.x / per_group) * p.G;
  const int rr = blockIdx.x % per_group;
  const int gs = min(p.G, p.BH - g0);
  const int jt = rr / gs;
  const int bh = g0 + rr % gs;
  const int hh = bh % p.H, hb = bh / p.H;  // TMA coordinates
  const int j0 = jt * kTile;
  const int i_first = p.causal ? jt : 0;
  const int n_loads = p.T - i_first;
  const float* vec = reinterpret_cast<const float*>(smem + L::VEC_OFF);  // nl, D, r, g [128] each
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, kStatusTimeout);
  };

  if (warp == kBobTmaWarp) {
    if (elect_one_sync()) {
      for (const CUtensorMap* m : {&tm_q, &tm_k, &tm_v, &tm_do, &tm_uq, &tm_uk, &tm_uv})
        prefetch_tensormap(m);
      mbar_arrive_expect_tx(&bars[O_RES], 4 * L::TILE);
      for (int c = 0; c < L::NCH; ++c) {
        tma_load_4d(smem + 0 * L::TILE + c * L::CHUNK, &tm_k, &bars[O_RES], c * L::CH, j0, hh, hb);
        tma_load_4d(smem + 1 * L::TILE + c * L::CHUNK, &tm_v, &bars[O_RES], c * L::CH, j0, hh, hb);
        tma_load_4d(smem + 2 * L::TILE + c * L::CHUNK, &tm_uk, &bars[O_RES], c * L::CH, j0, hh, hb);
        tma_load_4d(smem + 3 * L::TILE + c * L::CHUNK, &tm_uv, &bars[O_RES], c * L::CH, j0, hh, hb);
      }
      bool ok = true;
      int issued = 0;
      for (int n = 0; n < n_loads; ++n) {
        const int i0 = (i_first + n) * kTile;
        if (n > 0 && !(ok = mbar_wait(&bars[O_EMPTY], (n - 1) & 1, p.wait_cycles, abort_flag)))
          break;
        mbar_arrive_expect_tx(&bars[O_FULL], 3 * L::TILE + 4 * 512);
        for (int c = 0; c < L::NCH; ++c) {
          tma_load_4d(smem + 4 * L::TILE + c * L::CHUNK, &tm_q, &bars[O_FULL], c * L::CH, i0, hh, hb);
          tma_load_4d(smem + 5 * L::TILE + c * L::CHUNK, &tm_do, &bars[O_FULL], c * L::CH, i0, hh, hb);
          tma_load_4d(smem + 6 * L::TILE + c * L::CHUNK, &tm_uq, &bars[O_FULL], c * L::CH, i0, hh, hb);
        }
        const size_t v0 = static_cast<size_t>(bh) * p.Np + i0;
        bulk_load(smem + L::VEC_OFF + 0 * 512, p.nlse + v0, 512, &bars[O_FULL]);
        bulk_load(smem + L::VEC_OFF + 1 * 512, p.dvec + v0, 512, &bars[O_FULL]);
        bulk_load(smem + L::VEC_OFF + 2 * 512, p.r_pad + v0, 512, &bars[O_FULL]);
        bulk_load(smem + L::VEC_OFF + 3 * 512, p.g_pad + v0, 512, &bars[O_FULL]);
        ++issued;
      }
      if (!ok) fail();
      mbar_wait(&bars[O_RES], 0, p.wait_cycles, never);
      if (issued > 0) mbar_wait(&bars[O_FULL], (issued - 1) & 1, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp == kBobMmaWarp) {
    if (elect_one_sync()) {
      const uint32_t sK = sbase, sV = sbase + L::TILE, sUK = sbase + 2 * L::TILE;
      const uint32_t sUV = sbase + 3 * L::TILE, sQ = sbase + 4 * L::TILE;
      const uint32_t sDO = sbase + 5 * L::TILE, sUQ = sbase + 6 * L::TILE;
      auto wait = [&](int b, uint32_t parity) {
        return mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag);
      };
      bool ok = wait(O_RES, 0);
      int hn = 0;
      for (int n = 0; ok && n < n_loads; ++n) {
        if (!(ok = wait(O_FULL, n & 1))) break;
        tc_fence_after();
        for (int h = 0; h < 2; ++h, ++hn) {
          // S^T = K Q_h^T, dP^T = V dO_h^T, M^T = K U_Q,h^T + U_K Q_h^T, W^T = U_V dO_h^T
          issue_scores<D>(tmem, sK, sV, sK, sUK, sUV, sQ, sDO, sUQ, sQ, sDO,
                          static_cast<uint32_t>(64 * h * L::ROWB));
          mma_commit(&bars[O_SFULL]);
          if (!(ok = wait(O_EDONE, hn & 1))) break;
          tc_fence_after();
          // gK/s += dS^T U_Q,h + dS2^T Q_h;  gV += E^T dO_h
          const bool acc = hn > 0;
          issue_acc<D>(tmem, L::T_A0, L::T_S, sUQ, h, acc);
          issue_acc<D>(tmem, L::T_A0, L::T_DP, sQ, h, true);
          issue_acc<D>(tmem, L::T_A1, L::T_M, sDO, h, acc);
          mma_commit(&bars[O_ACC]);
          if (!(ok = wait(O_ACC, hn & 1))) break;
          tc_fence_after();
        }
        if (!ok) break;
        mma_commit(&bars[O_EMPTY]);
      }
      if (ok) {
        mma_commit(&bars[O_DONE]);
      } else {
        fail();
      }
      mma_commit(&bars[O_FINAL]);
      mbar_wait(&bars[O_FINAL], 0, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp < 8) {
    const int t = threadIdx.x & 127;  // TMEM lane: key j0 + t
    const int g = threadIdx.x >> 7;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = j0 + t;
    auto wait_w = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag));
    };
    bool ok = true;
    int hn = 0;
    for (int n = 0; ok && n < n_loads; ++n) {
      const int i0 = (i_first + n) * kTile;
      // the tile's query terms (-LSE log2 e, D, r, g) in shared memory
      if (!(ok = wait_w(O_FULL, n & 1))) break;
      for (int h = 0; h < 2; ++h, ++hn) {
        if (!(ok = wait_w(O_SFULL, hn & 1))) break;
        tc_fence_after();
        const int qb = 64 * h + 32 * g;  // first query (within the tile) of this thread's columns
        // columns u with u < thr are masked: keys past N mask every query;
        // the causal filter masks queries before the key
        int thr = 0;
        if (key >= p.N) thr = 32;
        else if (p.causal) thr = key - (i0 + qb);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          const uint32_t col = 32 * g + 16 * c;
          uint32_t s[16], dp[16], m[16], w[16];
          tmem_ld16(lane_base + L::T_S + col, s);
          tmem_ld16(lane_base + L::T_DP + col, dp);
          tmem_ld16(lane_base + L::T_M + col, m);
          tmem_ld16(lane_base + L::T_W + col, w);
          tmem_ld_wait(s, dp);
          tmem_ld_wait(m, w);
          uint32_t o_ds[8], o_ds2[8], o_e[8];
#pragma unroll
          for (int u = 0; u < 16; u += 2) {
            float ds[2], ds2[2], ev[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int uu = 16 * c + u + e;
              const int q = qb + uu;  // query within the tile
              const float nl = vec[0 * 128 + q], dv = vec[1 * 128 + q];
              const float rq = vec[2 * 128 + q], gq = vec[3 * 128 + q];
              float pp = ex2_approx(fmaf(__uint_as_float(s[u + e]), p.scale_log2, nl));
              if (uu < thr) pp = 0.f;
              const float mm = p.scale * __uint_as_float(m[u + e]);
              const float dpv = __uint_as_float(dp[u + e]);
              const float wv = __uint_as_float(w[u + e]);
              const float x = dpv - dv;
              ds[e] = pp * x;
              ds2[e] = pp * (fmaf(mm, x, fmaf(-rq, dpv, wv)) - gq);
              ev[e] = pp * (mm - rq);
            }
            o_ds[u / 2] = pack_bf16x2(ds[0], ds[1]);
            o_ds2[u / 2] = pack_bf16x2(ds2[0], ds2[1]);
            o_e[u / 2] = pack_bf16x2(ev[0], ev[1]);
          }
          const uint32_t oc = 32 * g + 8 * c;
          tmem_st8(lane_base + L::T_S + oc, o_ds);
          tmem_st8(lane_base + L::T_DP + oc, o_ds2);
          tmem_st8(lane_base + L::T_M + oc, o_e);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[O_EDONE]);
      }
    }
    if (ok) ok = wait_w(O_DONE, 0);
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      const bool key_ok = key < p.N && CSA_IN_BOUNDS(bh < p.BH && jt < p.T, p.status);
      const size_t orow = (static_cast<size_t>(bh) * p.N + (key_ok ? key : 0)) * D;
      // a key tile that meets no query tile (none, causal or not) still
      // accumulated at least one half: n_loads >= 1 always
      store_acc<D>(lane_base, L::T_A0, p.out0 + orow, key_ok, g, p.scale);
      store_acc<D>(lane_base, L::T_A1, p.out1 + orow, key_ok, g, 1.f);
    }
  }
  bob_teardown<D>(tmem);
}

template <int D>
cudaError_t launch_bob_bf16_d(const CUtensorMap (&maps)[7], const Workspace& ws, float* r_pad,
                              float* g_pad, void* gq, void* gk, void* gv, void* gdo, int BH, int H,
                              int N, bool causal, float scale, cudaStream_t s) {
  using L = BobLayout<D>;
  static_assert(L::ALLOC <= 232448, "shared memory window exceeds 227 KB");
  for (auto k : {bob_rows_bf16_kernel<D>, bob_cols_bf16_kernel<D>}) {
    const cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
  }
  BobParams p;
  p.nlse = ws.lse_pad;
  p.dvec = ws.d_pad;
  p.r_pad = r_pad;
  p.g_pad = g_pad;
  p.status = ws.status;
  p.N = N;
  p.Np = ws.Np;
  p.T = ws.Np / kTile;
  p.BH = BH;
  p.H = H;
  int dev = 0, l2 = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0)
    l2 = 126 << 20;
  // heads per group: the streamed side of a head (four or three [N][D] bf16
  // tensors) in about a third of L2
  const size_t head_bytes = static_cast<size_t>(ws.Np) * D * 2 * 4;
  p.G = static_cast<int>(std::max<size_t>(1, std::min<size_t>(BH, (l2 / 3) / head_bytes)));
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_cycles = kWaitLimitCycles;
  const unsigned grid = static_cast<unsigned>(p.T) * static_cast<unsigned>(BH);
  p.out0 = static_cast<__nv_bfloat16*>(gq);
  p.out1 = static_cast<__nv_bfloat16*>(gdo);
  bob_rows_bf16_kernel<D><<<grid, kBobThreads, L::ALLOC, s>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  p.out0 = static_cast<__nv_bfloat16*>(gk);
  p.out1 = static_cast<__nv_bfloat16*>(gv);
  bob_cols_bf16_kernel<D><<<grid, kBobThreads, L::ALLOC, s>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bob_bf16(const CUtensorMap (&maps)[7], const Workspace& ws, float* r_pad,
                            float* g_pad, void* gq, void* gk, void* gv, void* gdo, int BH, int H,
                            int N, int d, bool causal, float scale, cudaStream_t s) {
  switch (d) {
    case 32:
      return launch_bob_bf16_d<32>(maps, ws, r_pad, g_pad, gq, gk, gv, gdo, BH, H, N, causal,
                                   scale, s);
    case 64:
      return launch_bob_bf16_d<64>(maps, ws, r_pad, g_pad, gq, gk, gv, gdo, BH, H, N, causal,
                                   scale, s);
    case 128:
      return launch_bob_bf16_d<128>(maps, ws, r_pad, g_pad, gq, gk, gv, gdo, BH, H, N, causal,
                                    scale, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace csa
