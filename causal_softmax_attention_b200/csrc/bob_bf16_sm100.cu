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
// 128 x 32 block, so all of them run as tcgen05 MMAs:
//
//   rows kernel (one CTA per query tile, lanes = queries): key tiles in
//     32-key quarters; S, dP, M (two MMAs into one accumulator) and W into
//     four 32-column TMEM blocks. A first sweep over the key tiles forms the
//     row sums r and g in registers (and stores them for the columns
//     kernel); a second sweep writes dS, dS2, E and P as bf16 over the blocks
//     they came from and accumulates gQ / s += dS U_K + dS2 K and
//     gdO += E V + P U_V with TS MMAs (A from tensor memory, B the key rows
//     read MN-major).
//   columns kernel (one CTA per key tile, lanes = keys): query tiles in
//     32-query quarters; S^T, dP^T, M^T, W^T, then dS^T, dS2^T, E^T from the
//     stored r, g and gK / s += dS^T U_Q + dS2^T Q, gV += E^T dO.
//
// Score MMAs. An SS MMA (both operands in shared memory) of 128 x 32 x 16
// reads its 4 KB A slice for 32 output columns: shared memory, not the tensor
// core, sets its pace (40 cycles against 16). So wherever tensor memory has
// room, the resident tile's rows are copied into it once (packed bf16, lane =
// row) and the score MMAs run as TS MMAs that read only the 1 KB B slice. A
// sweep's TMEM layout (TmemLayout) holds, in order: those rows (when they
// fit), two or three sets of the four score blocks (128 columns each), and,
// in an accumulating sweep, the two fp32 accumulators (2 d columns). The
// rows kernel's first sweep has no accumulators and always runs TS; its
// second sweep and the columns kernel run TS at d <= 64 and SS at d = 128.
//
// Pipeline. The streamed side moves in 64-row halves through a ring of
// stages (two at d = 128, four below), so the next half loads while this one
// is used. The score MMAs of the next quarters run while the element-wise
// warps work on quarter k and the accumulating MMAs of earlier quarters
// finish. A set is overwritten only after the MMAs that read it (or, in the
// first sweep, the element-wise pass) have completed, so no ordering between
// MMAs of different accumulators is assumed; the rows kernel changes layout
// between its sweeps behind the row-sum exchange, when every first-sweep MMA
// and element-wise pass has ended.
//
// Warps (384 threads): 0-7 two element-wise warpgroups (thread t of group g
// owns TMEM lane t and the columns [16g, 16g+16) of each 32-column block);
// warp 8 issues the score MMAs, warp 10 the accumulating MMAs (two issuers,
// because an MMA issue waits while the tensor pipe's queue is full: one
// thread issuing both would hold each accumulation behind the next score
// batch), warp 9 the TMA loads; 11 idle. Every wait is bounded and reports a
// timeout. Nothing N x N is stored.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace {

using namespace sm100;

constexpr int kBobThreads = 384;
constexpr int kBobEThreads = 256;
constexpr int kBobMmaWarp = 8;   // score MMAs
constexpr int kBobTmaWarp = 9;
constexpr int kBobAccWarp = 10;  // accumulating MMAs
constexpr int kHalf = kBobBoxRows;  // streamed rows per stage
// Every wait here may sleep up to 20 us (it wakes when its phase completes):
// the warps that wait (MMA issuers, TMA producer, a group between quarters)
// share sub-partitions with the element-wise warps. Measured on one B200:
// 405 -> 412 TFLOP/s at d = 64, 501 -> 539 at d = 128.
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, uint64_t limit_cycles,
                                      const volatile int* abort) {
  return mbar_wait<kSuspendNs>(bar, parity, limit_cycles, abort);
}
constexpr int kQuarter = 32;        // score columns per block

template <int D>
struct BobLayout {
  static constexpr int CH = D >= 64 ? 64 : D;   // TMA box width (elements)
  static constexpr int NCH = D / CH;
  static constexpr int ROWB = CH * 2;
  static constexpr int CHUNK = kTile * ROWB;    // [128][CH]: a resident tile's chunk
  static constexpr int TILE = NCH * CHUNK;      // one resident [128][D] bf16 tile
  static constexpr int HCHUNK = kHalf * ROWB;   // [64][CH]: a streamed half's chunk
  static constexpr int HTILE = NCH * HCHUNK;    // one streamed [64][D] half
  static constexpr uint32_t SWZ = ROWB == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr int NST = D == 128 ? 2 : 4;  // stages in the ring
  // rows kernel: Q, dO, U_Q resident; stages of K, V, U_K, U_V halves, then
  // the row-sum exchange ([2 sums][2 groups][128] f32)
  static constexpr int ROWS_STAGE = 4 * HTILE;
  static constexpr int ROWS_END = 3 * TILE + NST * ROWS_STAGE;
  static constexpr int XCH_OFF = ROWS_END;
  // columns kernel: K, V, U_K, U_V resident; stages of Q, dO, U_Q halves and
  // the halves' per-query terms (-LSE log2 e, D, r, g: [4][64] f32)
  static constexpr int COLS_STAGE = 3 * HTILE + 4 * kHalf * 4;
  static constexpr int COLS_END = 4 * TILE + NST * COLS_STAGE;
  static constexpr int DATA_END =
      ROWS_END + 2048 > COLS_END ? ROWS_END + 2048 : COLS_END;
  static constexpr int BAR_OFF = DATA_END;
  static constexpr int MISC_OFF = BAR_OFF + 32 * 8;
  static constexpr int BYTES = MISC_OFF + 64;
  static_assert(HTILE % 1024 == 0 && COLS_STAGE % 1024 == 0, "swizzled stage alignment");
  // d = 128 fills the window but for 704 bytes (its base must then be
  // 1024-byte aligned, checked at run time); smaller d keep 1 KB of alignment
  // slack and at least ~118 KB, so that one CTA owns an SM's tensor memory
  static constexpr bool EXACT = D == 128;
  static constexpr int ALLOC =
      EXACT ? BYTES : ((BYTES + 1024) > 118 * 1024 ? BYTES + 1024 : 118 * 1024);
};

// A set of four 32-column score blocks.
constexpr uint32_t kTSet = 128;
constexpr uint32_t kTS = 0, kTDP = 32, kTM = 64, kTW = 96;
constexpr int kTCols = 512;

// One sweep's tensor memory: the resident rows for TS score MMAs (ROWS: Q,
// dO, U_Q; columns kernel: K, V, U_K, U_V -- tile x at column x d/2) when
// they fit beside two score sets and the accumulators, then NSET score sets,
// then (ACC) the two fp32 accumulators.
template <int D, bool ROWS, bool ACC>
struct TmemLayout {
  static constexpr int A_COLS = ((ROWS ? 3 : 4) * D / 2 + 31) / 32 * 32;
  static constexpr int ACC_COLS = ACC ? 2 * D : 0;
  static constexpr bool TS = A_COLS + 2 * static_cast<int>(kTSet) + ACC_COLS <= kTCols;
  static constexpr uint32_t SET0 = TS ? A_COLS : 0;
  static constexpr int NSET_FIT =
      (kTCols - static_cast<int>(SET0) - ACC_COLS) / static_cast<int>(kTSet);
  static constexpr int NSET = NSET_FIT > 3 ? 3 : NSET_FIT;
  static constexpr uint32_t T_A0 = SET0 + NSET * kTSet, T_A1 = T_A0 + D;
  static_assert(NSET >= 2, "two score sets at least");
  static_assert(!ACC || static_cast<int>(T_A1) + D <= kTCols, "TMEM columns exceeded");
};

// barrier slots: FULL and EMPTY per stage; SFULL / EDONE per score set of
// the accumulating sweep (and SFULL1 / EDONE1 of the rows kernel's first
// sweep); ACC per set
enum BobBar {
  O_RES = 0,
  O_FULL = 1,     // + stage (4 slots)
  O_EMPTY = 5,    // + stage (4 slots)
  O_SFULL = 9,    // + set (3 slots)
  O_EDONE = 12,   // + set (3 slots)
  O_SFULL1 = 15,  // + set (3 slots)
  O_EDONE1 = 18,  // + set (3 slots)
  O_ACC = 21,     // + set (3 slots)
  O_DONE = 24,
  O_XCH,
  O_FINAL,   // the score warp's MMAs have completed
  O_FINAL2,  // the accumulating warp's
  O_AREADY,  // the resident rows are in tensor memory
  O_COUNT
};
static_assert(O_COUNT <= 32, "barrier slots");

struct BobParams {
  const float* nlse;  // [BH][Np]: -LSE * log2(e), -inf past N
  const float* dvec;  // [BH][Np]: D, 0 past N
  float* r_pad;       // [BH][Np]: row scalar r (written by the rows kernel)
  float* g_pad;       // [BH][Np]: row scalar g
  // rows kernel: Q, dO, U_Q; columns kernel: K, V, U_K, U_V ([BH][N][D])
  const __nv_bfloat16* res[4];
  __nv_bfloat16* out0;  // rows kernel: gQ; columns kernel: gK   ([BH][N][D])
  __nv_bfloat16* out1;  // rows kernel: gdO; columns kernel: gV
  int* status;
  int N, Np, T, BH, H, G, causal;  // H splits bh into the tensor maps' (head, batch)
  float scale, scale_log2;
  uint64_t wait_cycles;
  int inject_fault;  // rows kernel: never signal the first score quarter (the timeout test)
};

// K-major operand slice kk (16 elements of the contraction) of a [rows][D]
// region whose CH-wide chunks lie `chunk` bytes apart.
template <int D>
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int chunk, int kk) {
  using L = BobLayout<D>;
  const int e = kk * 16;
  return smem_desc(base + (e / L::CH) * chunk + (e % L::CH) * 2, 16, 8 * L::ROWB, L::SWZ);
}
// The same region read MN-major: its rows are the contraction (16 from
// `row_base`), its D channels the N dimension.
template <int D>
__device__ __forceinline__ uint64_t desc_mn(uint32_t row_base, int chunk) {
  using L = BobLayout<D>;
  return smem_desc(row_base, chunk, 8 * L::ROWB, L::SWZ);
}

// Score MMAs of one quarter into the set at `set`: four [128 x 32] fp32 blocks
//   S = A0 B0^T,  dP = A1 B1^T,  M = A2 B2^T + A3 B3^T,  W = A4 B4^T
// with B the quarter's 32 rows of a streamed half. TS: the A operands are
// resident rows in tensor memory (addresses); SS: resident [128][D] tiles in
// shared memory.
template <int D, bool TS>
__device__ __forceinline__ void issue_scores(uint32_t set, const uint32_t (&a)[5],
                                             const uint32_t (&b)[5]) {
  using L = BobLayout<D>;
  constexpr uint32_t ID = idesc_bf16(128, kQuarter, false, false);
  auto one = [&](uint32_t dst, int x, int kk, uint32_t accumulate) {
    const uint64_t bd = desc_k<D>(b[x], L::HCHUNK, kk);
    if (TS)
      mma_ts(dst, a[x] + 8 * kk, bd, ID, accumulate);
    else
      mma_ss(dst, desc_k<D>(a[x], L::CHUNK, kk), bd, ID, accumulate);
  };
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t c = kk > 0;
    one(set + kTS, 0, kk, c);
    one(set + kTDP, 1, kk, c);
    one(set + kTM, 2, kk, c);
    one(set + kTW, 4, kk, c);
  }
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) one(set + kTM, 3, kk, 1);
}

// acc (+)= [packed bf16 block at `blk`] x B, B the quarter's 32 rows of a
// streamed half (from `b`), read MN-major (K = those rows, N = D channels).
// Group g's 16 elements of a block sit packed in its columns [16g, 16g+8),
// so contraction slice kk is group kk's.
template <int D>
__device__ __forceinline__ void issue_acc(uint32_t tmem, uint32_t acc, uint32_t blk, uint32_t b,
                                          bool accumulate) {
  using L = BobLayout<D>;
  constexpr uint32_t ID = idesc_bf16(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < kQuarter / 16; ++kk)
    mma_ts(tmem + acc, tmem + blk + 16 * kk, desc_mn<D>(b + 16 * kk * L::ROWB, L::HCHUNK), ID,
           (accumulate || kk > 0) ? 1u : 0u);
}

// The score warp's loop over n_q quarters, shared by both kernels: scores(k)
// issues quarter k's score MMAs (it waits for the quarter's stage itself).
// Quarters before first_acc form the rows kernel's first sweep (sets of
// TmemLayout<.., false>), the rest the accumulating sweep. Before quarter k
// overwrites the set of the sweep's quarter k - NSET, what read it must have
// completed: its accumulating MMAs, or in the first sweep its element-wise
// pass. First-sweep stages are released here, after their second quarter.
template <int D, bool ROWS, class Scores>
__device__ __forceinline__ bool bob_score_loop(uint64_t* bars, int n_q, int first_acc,
                                               uint64_t wait_cycles, volatile int* abort_flag,
                                               Scores scores) {
  using L = BobLayout<D>;
  using T1 = TmemLayout<D, ROWS, false>;
  using T2 = TmemLayout<D, ROWS, true>;
  auto wait = [&](int b, uint32_t parity) {
    return bwait(&bars[b], parity, wait_cycles, abort_flag);
  };
  for (int k = 0; k < n_q; ++k) {
    if (k < first_acc) {
      const int kp = k - T1::NSET;
      if (kp >= 0 && !wait(O_EDONE1 + kp % T1::NSET, (kp / T1::NSET) & 1)) return false;
    } else {
      // the row-sum exchange: every first-sweep pass has ended, so every
      // first-sweep MMA has completed and tensor memory takes this sweep's
      // layout
      if (k == first_acc && first_acc > 0 && !wait(O_XCH, 0)) return false;
      const int kp = k - first_acc - T2::NSET;
      if (kp >= 0 && !wait(O_ACC + kp % T2::NSET, (kp / T2::NSET) & 1)) return false;
    }
    if (!scores(k)) return false;
    if ((k & 1) && k < first_acc) mma_commit(&bars[O_EMPTY + (k >> 1) % L::NST]);
  }
  return true;
}

// The accumulating warp's loop over quarters first_acc .. n_q - 1: once
// quarter k's element-wise pass is done, acc(k, set, accumulate) issues its
// MMAs; their completion releases the set (ACC) and, after a stage's second
// quarter, the stage. Its own issue queue, so that these MMAs never wait
// behind a score batch that cannot be issued yet.
template <int D, bool ROWS, class Acc>
__device__ __forceinline__ bool bob_acc_loop(uint64_t* bars, int n_q, int first_acc,
                                             uint64_t wait_cycles, volatile int* abort_flag,
                                             Acc acc) {
  using L = BobLayout<D>;
  using T2 = TmemLayout<D, ROWS, true>;
  for (int k = first_acc; k < n_q; ++k) {
    const int kl = k - first_acc, b = kl % T2::NSET;
    if (!bwait(&bars[O_EDONE + b], (kl / T2::NSET) & 1, wait_cycles, abort_flag))
      return false;
    tc_fence_after();
    acc(k, T2::SET0 + static_cast<uint32_t>(b) * kTSet, kl > 0);
    mma_commit(&bars[O_ACC + b]);
    if (k & 1) mma_commit(&bars[O_EMPTY + (k >> 1) % L::NST]);
  }
  return true;
}

// Rows i0 + t (lanes) of NT resident tiles into tensor memory as packed bf16
// pairs, tile x at columns [x D/2, (x+1) D/2): the A operands of TS score
// MMAs. Group g copies channels [g D/2, (g+1) D/2) of each; rows at or past
// N are zeros (the tiles' TMA copies read them as zeros too).
template <int D, int NT>
__device__ __forceinline__ void load_rows_to_tmem(uint32_t lane_base,
                                                  const __nv_bfloat16* const (&src)[4],
                                                  size_t row_elem, bool row_ok, int g) {
  constexpr int W = D / 4;  // 32-bit columns per group per tile
#pragma unroll
  for (int x = 0; x < NT; ++x) {
    uint32_t v[W];
    const uint4* s4 = reinterpret_cast<const uint4*>(src[x] + row_elem + g * (D / 2));
#pragma unroll
    for (int i = 0; i < W / 4; ++i) {
      const uint4 q = row_ok ? __ldg(s4 + i) : make_uint4(0u, 0u, 0u, 0u);
      v[4 * i + 0] = q.x;
      v[4 * i + 1] = q.y;
      v[4 * i + 2] = q.z;
      v[4 * i + 3] = q.w;
    }
    const uint32_t col = lane_base + x * (D / 2) + g * W;
    if constexpr (W == 32)
      tmem_st32(col, v);
    else if constexpr (W == 16)
      tmem_st16(col, v);
    else
      tmem_st8(col, v);
  }
  tmem_st_wait();
}

// First-sweep row sums over 16 columns: r += P M, g += P (M dP + W) (M
// already scaled), as packed pairs. Columns u >= lim are masked.
template <bool MASK>
__device__ __forceinline__ void rows_sums(const uint32_t (&s)[16], const uint32_t (&dp)[16],
                                          const uint32_t (&m)[16], const uint32_t (&w)[16],
                                          uint64_t sl2, uint64_t nl2, uint64_t sc2, int lim,
                                          uint64_t& r2, uint64_t& g2) {
#pragma unroll
  for (int u = 0; u < 16; u += 2) {
    float2 a = f2_split(fma2(f2(__uint_as_float(s[u]), __uint_as_float(s[u + 1])), sl2, nl2));
    if (MASK) {
      if (u >= lim) a.x = -INFINITY;
      if (u + 1 >= lim) a.y = -INFINITY;
    }
    const uint64_t pp = f2(ex2_approx(a.x), ex2_approx(a.y));
    const uint64_t mm = mul2(f2(__uint_as_float(m[u]), __uint_as_float(m[u + 1])), sc2);
    const uint64_t dpv = f2(__uint_as_float(dp[u]), __uint_as_float(dp[u + 1]));
    const uint64_t wv = f2(__uint_as_float(w[u]), __uint_as_float(w[u + 1]));
    r2 = fma2(pp, mm, r2);
    g2 = fma2(pp, fma2(mm, dpv, wv), g2);
  }
}

// Second-pass products of 16 columns, packed to bf16 pairs: dS, dS2, E (and
// P when ROWS). nl2 / dv2 / r2 / g2 give each column's -LSE log2 e, D, r, g:
// one value for both lanes of a pair (rows kernel) or per column (columns
// kernel, through `vec`). Columns u >= lim (rows) or u < lim (columns) are
// masked.
template <bool MASK, bool ROWS>
__device__ __forceinline__ void second_pass(const uint32_t (&s)[16], const uint32_t (&dp)[16],
                                            const uint32_t (&m)[16], const uint32_t (&w)[16],
                                            uint64_t sl2, uint64_t sc2, uint64_t nl2,
                                            uint64_t dv2, uint64_t r2, uint64_t g2,
                                            const float* vec, int lim, uint32_t (&o_ds)[8],
                                            uint32_t (&o_ds2)[8], uint32_t (&o_e)[8],
                                            uint32_t (&o_p)[8]) {
#pragma unroll
  for (int u = 0; u < 16; u += 2) {
    if (!ROWS) {
      const float2 nv = *reinterpret_cast<const float2*>(vec + 0 * kHalf + u);
      const float2 dvv = *reinterpret_cast<const float2*>(vec + 1 * kHalf + u);
      const float2 rv = *reinterpret_cast<const float2*>(vec + 2 * kHalf + u);
      const float2 gv = *reinterpret_cast<const float2*>(vec + 3 * kHalf + u);
      nl2 = f2(nv.x, nv.y);
      dv2 = f2(dvv.x, dvv.y);
      r2 = f2(rv.x, rv.y);
      g2 = f2(gv.x, gv.y);
    }
    float2 a = f2_split(fma2(f2(__uint_as_float(s[u]), __uint_as_float(s[u + 1])), sl2, nl2));
    if (MASK) {
      if (ROWS ? u >= lim : u < lim) a.x = -INFINITY;
      if (ROWS ? u + 1 >= lim : u + 1 < lim) a.y = -INFINITY;
    }
    const uint64_t pp = f2(ex2_approx(a.x), ex2_approx(a.y));
    const uint64_t mm = mul2(f2(__uint_as_float(m[u]), __uint_as_float(m[u + 1])), sc2);
    const uint64_t dpv = f2(__uint_as_float(dp[u]), __uint_as_float(dp[u + 1]));
    const uint64_t wv = f2(__uint_as_float(w[u]), __uint_as_float(w[u + 1]));
    const uint64_t x = sub2(dpv, dv2);
    // dS2 = P (M (dP - D) + W - (r dP + g))
    const uint64_t t = sub2(fma2(mm, x, wv), fma2(r2, dpv, g2));
    const float2 ds = f2_split(mul2(pp, x));
    const float2 ds2 = f2_split(mul2(pp, t));
    const float2 ev = f2_split(mul2(pp, sub2(mm, r2)));
    o_ds[u / 2] = pack_bf16x2(ds.x, ds.y);
    o_ds2[u / 2] = pack_bf16x2(ds2.x, ds2.y);
    o_e[u / 2] = pack_bf16x2(ev.x, ev.y);
    if (ROWS) {
      const float2 pv = f2_split(pp);
      o_p[u / 2] = pack_bf16x2(pv.x, pv.y);
    }
  }
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
    for (int s = 0; s < L::NST; ++s) {
      mbar_init(&bars[O_FULL + s], 1);
      mbar_init(&bars[O_EMPTY + s], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bars[O_SFULL + b], 1);
      mbar_init(&bars[O_EDONE + b], kBobEThreads);
      mbar_init(&bars[O_SFULL1 + b], 1);
      mbar_init(&bars[O_EDONE1 + b], kBobEThreads);
      mbar_init(&bars[O_ACC + b], 1);
    }
    mbar_init(&bars[O_DONE], 1);
    mbar_init(&bars[O_XCH], kBobEThreads);
    mbar_init(&bars[O_FINAL], 1);
    mbar_init(&bars[O_FINAL2], 1);
    mbar_init(&bars[O_AREADY], kBobEThreads);
    *abort_flag = 0;
    *const_cast<volatile int*>(never) = 0;
    fence_barrier_init();
  }
  if ((threadIdx.x >> 5) == 0) {
    tmem_alloc(tmem_slot, kTCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tmem = *tmem_slot;
  return true;
}

__device__ __forceinline__ void bob_teardown(uint32_t tmem) {
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTCols);
  }
}

// The TMA warp's loop: units u = 0 .. n_units - 1 into the ring (stage
// u % NST, reused once the MMAs of unit u - NST have completed); load(u, st,
// bar) issues unit u's copies into the stage at `st`. Before the CTA exits,
// every copy issued has landed (bounded waits).
template <int D, class Load>
__device__ __forceinline__ bool bob_load_loop(uint64_t* bars, int n_units, uint64_t wait_cycles,
                                              volatile int* abort_flag, const volatile int* never,
                                              Load load) {
  using L = BobLayout<D>;
  bool ok = true;
  int issued = 0;
  for (int u = 0; u < n_units; ++u) {
    const int s = u % L::NST;
    if (u >= L::NST &&
        !(ok = bwait(&bars[O_EMPTY + s], ((u / L::NST) - 1) & 1, wait_cycles, abort_flag)))
      break;
    load(u, s, &bars[O_FULL + s]);
    ++issued;
  }
  bwait(&bars[O_RES], 0, wait_cycles, never);
  for (int u = max(0, issued - L::NST); u < issued; ++u)
    bwait(&bars[O_FULL + u % L::NST], (u / L::NST) & 1, wait_cycles, never);
  return ok;
}

// ============================================================== rows kernel
// Resident: Q_i, dO_i, U_Q,i. Streamed halves: K_j, V_j, U_K,j, U_V,j.
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
  using T1 = TmemLayout<D, true, false>;  // first sweep
  using T2 = TmemLayout<D, true, true>;   // second (accumulating) sweep
  static_assert(T1::TS, "the first sweep reads Q, dO, U_Q from tensor memory");
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
  const int n_units = 4 * n_kt;                 // halves over two sweeps
  const int n_q = 2 * n_units;                  // quarters
  const int first_acc = 4 * n_kt;               // the second sweep's first quarter
  // key row of unit u's half
  auto unit_key = [&](int u) { return ((u >> 1) % n_kt) * kTile + kHalf * (u & 1); };
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
      for (int c = 0; c < L::NCH; ++c)
        for (int hr = 0; hr < 2; ++hr) {
          const int off = c * L::CHUNK + hr * L::HCHUNK, row = i0 + kHalf * hr;
          tma_load_4d(smem + 0 * L::TILE + off, &tm_q, &bars[O_RES], c * L::CH, row, hh, hb);
          tma_load_4d(smem + 1 * L::TILE + off, &tm_do, &bars[O_RES], c * L::CH, row, hh, hb);
          tma_load_4d(smem + 2 * L::TILE + off, &tm_uq, &bars[O_RES], c * L::CH, row, hh, hb);
        }
      const bool ok = bob_load_loop<D>(
          bars, n_units, p.wait_cycles, abort_flag, never, [&](int u, int s, uint64_t* bar) {
            uint8_t* st = smem + 3 * L::TILE + s * L::ROWS_STAGE;
            const int j = unit_key(u);
            mbar_arrive_expect_tx(bar, 4 * L::HTILE);
            for (int c = 0; c < L::NCH; ++c) {
              uint8_t* dst = st + c * L::HCHUNK;
              tma_load_4d(dst + 0 * L::HTILE, &tm_k, bar, c * L::CH, j, hh, hb);
              tma_load_4d(dst + 1 * L::HTILE, &tm_v, bar, c * L::CH, j, hh, hb);
              tma_load_4d(dst + 2 * L::HTILE, &tm_uk, bar, c * L::CH, j, hh, hb);
              tma_load_4d(dst + 3 * L::HTILE, &tm_uv, bar, c * L::CH, j, hh, hb);
            }
          });
      if (!ok) fail();
    }
    __syncwarp();
  } else if (warp == kBobMmaWarp || warp == kBobAccWarp) {
    // ------------------------------------------------ MMA issuers
    if (elect_one_sync()) {
      // A operands: Q, dO, U_Q, Q, dO (S, dP, M's two products, W)
      const uint32_t sQ = sbase, sDO = sbase + L::TILE, sUQ = sbase + 2 * L::TILE;
      const uint32_t a_smem[5] = {sQ, sDO, sUQ, sQ, sDO};
      const uint32_t tQ = tmem, tDO = tmem + D / 2, tUQ = tmem + D;
      const uint32_t a_tmem[5] = {tQ, tDO, tUQ, tQ, tDO};
      // the quarter's rows of its stage: K, V, U_K, U_V at HTILE steps
      auto qrows = [&](int k) {
        return sbase + 3 * L::TILE + ((k >> 1) % L::NST) * L::ROWS_STAGE +
               kQuarter * (k & 1) * L::ROWB;
      };
      auto scores = [&](int k) {
        const int u = k >> 1;
        if ((k & 1) == 0 &&
            !bwait(&bars[O_FULL + u % L::NST], (u / L::NST) & 1, p.wait_cycles, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t st = qrows(k);
        // S = Q K^T, dP = dO V^T, M = U_Q K^T + Q U_K^T, W = dO U_V^T
        const uint32_t b[5] = {st, st + L::HTILE, st, st + 2 * L::HTILE, st + 3 * L::HTILE};
        if (k < first_acc) {
          const int s = k % T1::NSET;
          issue_scores<D, T1::TS>(tmem + T1::SET0 + s * kTSet, a_tmem, b);
          if (!(p.inject_fault && k == 0)) mma_commit(&bars[O_SFULL1 + s]);
        } else {
          const int s = (k - first_acc) % T2::NSET;
          issue_scores<D, T2::TS>(tmem + T2::SET0 + s * kTSet, T2::TS ? a_tmem : a_smem, b);
          mma_commit(&bars[O_SFULL + s]);
        }
        return true;
      };
      auto acc = [&](int k, uint32_t set, bool accumulate) {
        const uint32_t st = qrows(k);
        // gQ/s += dS U_K + dS2 K;  gdO += E V + P U_V
        issue_acc<D>(tmem, T2::T_A0, set + kTS, st + 2 * L::HTILE, accumulate);
        issue_acc<D>(tmem, T2::T_A0, set + kTDP, st, true);
        issue_acc<D>(tmem, T2::T_A1, set + kTM, st + L::HTILE, accumulate);
        issue_acc<D>(tmem, T2::T_A1, set + kTW, st + 3 * L::HTILE, true);
      };
      if (warp == kBobMmaWarp) {
        if (!(bwait(&bars[O_RES], 0, p.wait_cycles, abort_flag) &&
              bwait(&bars[O_AREADY], 0, p.wait_cycles, abort_flag) &&
              bob_score_loop<D, true>(bars, n_q, first_acc, p.wait_cycles, abort_flag, scores)))
          fail();
      } else {
        // the row-sum exchange: the second sweep's layout is in force
        if (bwait(&bars[O_XCH], 0, p.wait_cycles, abort_flag) &&
            bob_acc_loop<D, true>(bars, n_q, first_acc, p.wait_cycles, abort_flag, acc))
          mma_commit(&bars[O_DONE]);
        else
          fail();
      }
      const int fin = warp == kBobMmaWarp ? O_FINAL : O_FINAL2;
      mma_commit(&bars[fin]);
      bwait(&bars[fin], 0, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------ element-wise warpgroups
    const int t = threadIdx.x & 127;  // TMEM lane: query row i0 + t
    const int g = threadIdx.x >> 7;   // columns [16g, 16g+16) of each block
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int row = i0 + t;
    const bool row_ok = row < p.N && CSA_IN_BOUNDS(bh < p.BH && it_q < p.T, p.status);
    const size_t vrow = static_cast<size_t>(bh) * p.Np + row;
    const size_t orow = (static_cast<size_t>(bh) * p.N + (row_ok ? row : 0)) * D;
    // Q, dO, U_Q rows into tensor memory for the TS score MMAs
    load_rows_to_tmem<D, 3>(lane_base, p.res, orow, row_ok, g);
    tc_fence_before();
    mbar_arrive(&bars[O_AREADY]);
    const float nl = p.nlse[vrow];
    const float dv = p.dvec[vrow];
    float* xch = reinterpret_cast<float*>(smem + L::XCH_OFF);  // [2 sums][2 groups][128]
    auto wait_w = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, bwait(&bars[b], parity, p.wait_cycles, abort_flag));
    };
    const uint64_t sl2 = f2(p.scale_log2, p.scale_log2), sc2 = f2(p.scale, p.scale);
    const uint64_t nl2 = f2(nl, nl), dv2 = f2(dv, dv);
    uint64_t r_acc = f2(0.f, 0.f), g_acc = f2(0.f, 0.f);  // this group's partial row sums
    uint64_t r2 = 0, g2 = 0;                                // the row scalars (second sweep)
    bool ok = true;
    for (int k = 0; ok && k < n_q; ++k) {
      if (k == first_acc) {
        // both groups' partial sums -> r, g of the row (a bounded barrier
        // wait, so that a timed-out group cannot hold the other forever)
        const float2 rp = f2_split(r_acc), gp = f2_split(g_acc);
        xch[(0 * 2 + g) * 128 + t] = rp.x + rp.y;
        xch[(1 * 2 + g) * 128 + t] = gp.x + gp.y;
        mbar_arrive(&bars[O_XCH]);
        if (!(ok = wait_w(O_XCH, 0))) break;
        const float rr_ = xch[(0 * 2 + 0) * 128 + t] + xch[(0 * 2 + 1) * 128 + t];
        const float gg_ = xch[(1 * 2 + 0) * 128 + t] + xch[(1 * 2 + 1) * 128 + t] - 2.f * rr_ * dv;
        r2 = f2(rr_, rr_);
        g2 = f2(gg_, gg_);
        if (g == 0 && CSA_IN_BOUNDS(row < p.Np && bh < p.BH, p.status)) {
          p.r_pad[vrow] = rr_;
          p.g_pad[vrow] = gg_;
        }
      }
      const bool second = k >= first_acc;
      const int kl = second ? k - first_acc : k;
      const int nset = second ? T2::NSET : T1::NSET;
      const int b = kl % nset;
      if (!(ok = wait_w((second ? O_SFULL : O_SFULL1) + b, (kl / nset) & 1))) break;
      tc_fence_after();
      const int kb = unit_key(k >> 1) + kQuarter * (k & 1) + 16 * g;  // first key of these 16 columns
      int lim = p.N - kb;                                       // columns u >= lim are masked
      if (p.causal && row - kb + 1 < lim) lim = row - kb + 1;
      const uint32_t col = lane_base + (second ? T2::SET0 : T1::SET0) + b * kTSet + 16 * g;
      // the masked pass is taken by the whole warp whenever one lane needs
      // it: the TMEM accesses that follow are warp-collective, and a per-lane
      // choice lets the compiler issue them from divergent paths
      uint32_t s[16], dp[16], m[16], w[16];
      tmem_ld16(col + kTS, s);
      tmem_ld16(col + kTDP, dp);
      tmem_ld16(col + kTM, m);
      tmem_ld16(col + kTW, w);
      tmem_ld_wait(s, dp);
      tmem_ld_wait(m, w);
      if (!second) {
        if (__any_sync(0xffffffffu, lim < 16))
          rows_sums<true>(s, dp, m, w, sl2, nl2, sc2, lim, r_acc, g_acc);
        else
          rows_sums<false>(s, dp, m, w, sl2, nl2, sc2, lim, r_acc, g_acc);
      } else {
        uint32_t o_ds[8], o_ds2[8], o_e[8], o_p[8];
        if (__any_sync(0xffffffffu, lim < 16))
          second_pass<true, true>(s, dp, m, w, sl2, sc2, nl2, dv2, r2, g2, nullptr, lim, o_ds,
                                  o_ds2, o_e, o_p);
        else
          second_pass<false, true>(s, dp, m, w, sl2, sc2, nl2, dv2, r2, g2, nullptr, lim, o_ds,
                                   o_ds2, o_e, o_p);
        // packed pairs into the first 8 of the group's 16 columns of each block
        tmem_st8(col + kTS, o_ds);
        tmem_st8(col + kTDP, o_ds2);
        tmem_st8(col + kTM, o_e);
        tmem_st8(col + kTW, o_p);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bars[(second ? O_EDONE : O_EDONE1) + b]);
    }
    if (ok) ok = wait_w(O_DONE, 0);
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      store_acc<D>(lane_base, T2::T_A0, p.out0 + orow, row_ok, g, p.scale);
      store_acc<D>(lane_base, T2::T_A1, p.out1 + orow, row_ok, g, 1.f);
    }
  }
  bob_teardown(tmem);
}

// ============================================================== columns kernel
// Resident: K_j, V_j, U_K,j, U_V,j. Streamed halves: Q_i, dO_i, U_Q,i and
// their -LSE log2 e, D, r, g.
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
  using T2 = TmemLayout<D, false, true>;
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
  const int n_units = 2 * (p.T - i_first);  // query halves
  const int n_q = 2 * n_units;
  auto unit_query = [&](int u) { return (i_first + (u >> 1)) * kTile + kHalf * (u & 1); };
  auto stage_off = [&](int s) { return 4 * L::TILE + s * L::COLS_STAGE; };
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, kStatusTimeout);
  };

  if (warp == kBobTmaWarp) {
    if (elect_one_sync()) {
      for (const CUtensorMap* m : {&tm_q, &tm_k, &tm_v, &tm_do, &tm_uq, &tm_uk, &tm_uv})
        prefetch_tensormap(m);
      mbar_arrive_expect_tx(&bars[O_RES], 4 * L::TILE);
      for (int c = 0; c < L::NCH; ++c)
        for (int hr = 0; hr < 2; ++hr) {
          const int off = c * L::CHUNK + hr * L::HCHUNK, row = j0 + kHalf * hr;
          tma_load_4d(smem + 0 * L::TILE + off, &tm_k, &bars[O_RES], c * L::CH, row, hh, hb);
          tma_load_4d(smem + 1 * L::TILE + off, &tm_v, &bars[O_RES], c * L::CH, row, hh, hb);
          tma_load_4d(smem + 2 * L::TILE + off, &tm_uk, &bars[O_RES], c * L::CH, row, hh, hb);
          tma_load_4d(smem + 3 * L::TILE + off, &tm_uv, &bars[O_RES], c * L::CH, row, hh, hb);
        }
      const bool ok = bob_load_loop<D>(
          bars, n_units, p.wait_cycles, abort_flag, never, [&](int u, int s, uint64_t* bar) {
            uint8_t* st = smem + stage_off(s);
            const int i = unit_query(u);
            mbar_arrive_expect_tx(bar, 3 * L::HTILE + 4 * kHalf * 4);
            for (int c = 0; c < L::NCH; ++c) {
              uint8_t* dst = st + c * L::HCHUNK;
              tma_load_4d(dst + 0 * L::HTILE, &tm_q, bar, c * L::CH, i, hh, hb);
              tma_load_4d(dst + 1 * L::HTILE, &tm_do, bar, c * L::CH, i, hh, hb);
              tma_load_4d(dst + 2 * L::HTILE, &tm_uq, bar, c * L::CH, i, hh, hb);
            }
            const size_t v0 = static_cast<size_t>(bh) * p.Np + i;
            uint8_t* vd = st + 3 * L::HTILE;
            bulk_load(vd + 0 * kHalf * 4, p.nlse + v0, kHalf * 4, bar);
            bulk_load(vd + 1 * kHalf * 4, p.dvec + v0, kHalf * 4, bar);
            bulk_load(vd + 2 * kHalf * 4, p.r_pad + v0, kHalf * 4, bar);
            bulk_load(vd + 3 * kHalf * 4, p.g_pad + v0, kHalf * 4, bar);
          });
      if (!ok) fail();
    }
    __syncwarp();
  } else if (warp == kBobMmaWarp || warp == kBobAccWarp) {
    if (elect_one_sync()) {
      // A operands: K, V, K, U_K, U_V (S^T, dP^T, M^T's two products, W^T)
      const uint32_t sK = sbase, sV = sbase + L::TILE, sUK = sbase + 2 * L::TILE;
      const uint32_t sUV = sbase + 3 * L::TILE;
      const uint32_t a_smem[5] = {sK, sV, sK, sUK, sUV};
      const uint32_t tK = tmem, tV = tmem + D / 2, tUK = tmem + D, tUV = tmem + 3 * D / 2;
      const uint32_t a_tmem[5] = {tK, tV, tK, tUK, tUV};
      auto qrows = [&](int k) {
        return sbase + stage_off((k >> 1) % L::NST) + kQuarter * (k & 1) * L::ROWB;
      };
      auto scores = [&](int k) {
        const int u = k >> 1;
        if ((k & 1) == 0 &&
            !bwait(&bars[O_FULL + u % L::NST], (u / L::NST) & 1, p.wait_cycles, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t st = qrows(k);
        // S^T = K Q^T, dP^T = V dO^T, M^T = K U_Q^T + U_K Q^T, W^T = U_V dO^T
        const uint32_t b[5] = {st, st + L::HTILE, st + 2 * L::HTILE, st, st + L::HTILE};
        const int s = k % T2::NSET;
        issue_scores<D, T2::TS>(tmem + T2::SET0 + s * kTSet, T2::TS ? a_tmem : a_smem, b);
        mma_commit(&bars[O_SFULL + s]);
        return true;
      };
      auto acc = [&](int k, uint32_t set, bool accumulate) {
        const uint32_t st = qrows(k);
        // gK/s += dS^T U_Q + dS2^T Q;  gV += E^T dO
        issue_acc<D>(tmem, T2::T_A0, set + kTS, st + 2 * L::HTILE, accumulate);
        issue_acc<D>(tmem, T2::T_A0, set + kTDP, st, true);
        issue_acc<D>(tmem, T2::T_A1, set + kTM, st + L::HTILE, accumulate);
      };
      if (warp == kBobMmaWarp) {
        if (!(bwait(&bars[O_RES], 0, p.wait_cycles, abort_flag) &&
              (!T2::TS || bwait(&bars[O_AREADY], 0, p.wait_cycles, abort_flag)) &&
              bob_score_loop<D, false>(bars, n_q, 0, p.wait_cycles, abort_flag, scores)))
          fail();
      } else {
        if (bob_acc_loop<D, false>(bars, n_q, 0, p.wait_cycles, abort_flag, acc))
          mma_commit(&bars[O_DONE]);
        else
          fail();
      }
      const int fin = warp == kBobMmaWarp ? O_FINAL : O_FINAL2;
      mma_commit(&bars[fin]);
      bwait(&bars[fin], 0, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp < 8) {
    const int t = threadIdx.x & 127;  // TMEM lane: key j0 + t
    const int g = threadIdx.x >> 7;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = j0 + t;
    const bool key_ok = key < p.N && CSA_IN_BOUNDS(bh < p.BH && jt < p.T, p.status);
    const size_t orow = (static_cast<size_t>(bh) * p.N + (key_ok ? key : 0)) * D;
    if constexpr (T2::TS) {
      // K, V, U_K, U_V rows into tensor memory for the TS score MMAs
      load_rows_to_tmem<D, 4>(lane_base, p.res, orow, key_ok, g);
      tc_fence_before();
      mbar_arrive(&bars[O_AREADY]);
    }
    auto wait_w = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, bwait(&bars[b], parity, p.wait_cycles, abort_flag));
    };
    const uint64_t sl2 = f2(p.scale_log2, p.scale_log2), sc2 = f2(p.scale, p.scale);
    bool ok = true;
    for (int k = 0; ok && k < n_q; ++k) {
      const int u = k >> 1, b = k % T2::NSET;
      // the half's query terms (-LSE log2 e, D, r, g) land with its tiles
      if ((k & 1) == 0 && !(ok = wait_w(O_FULL + u % L::NST, (u / L::NST) & 1))) break;
      if (!(ok = wait_w(O_SFULL + b, (k / T2::NSET) & 1))) break;
      tc_fence_after();
      const int qo = kQuarter * (k & 1) + 16 * g;  // first query (within the half) of these columns
      const float* vec =
          reinterpret_cast<const float*>(smem + stage_off(u % L::NST) + 3 * L::HTILE) + qo;
      // columns u < thr are masked: keys past N mask every query; the causal
      // filter masks queries before the key
      int thr = 0;
      if (key >= p.N) thr = 16;
      else if (p.causal) thr = key - (unit_query(u) + qo);
      const uint32_t col = lane_base + T2::SET0 + b * kTSet + 16 * g;
      // the masked pass is taken by the whole warp whenever one lane needs
      // it: the TMEM accesses that follow are warp-collective, and a per-lane
      // choice lets the compiler issue them from divergent paths
      uint32_t s[16], dp[16], m[16], w[16];
      tmem_ld16(col + kTS, s);
      tmem_ld16(col + kTDP, dp);
      tmem_ld16(col + kTM, m);
      tmem_ld16(col + kTW, w);
      tmem_ld_wait(s, dp);
      tmem_ld_wait(m, w);
      uint32_t o_ds[8], o_ds2[8], o_e[8], o_p[8];
      if (__any_sync(0xffffffffu, thr > 0))
        second_pass<true, false>(s, dp, m, w, sl2, sc2, 0, 0, 0, 0, vec, thr, o_ds, o_ds2, o_e,
                                 o_p);
      else
        second_pass<false, false>(s, dp, m, w, sl2, sc2, 0, 0, 0, 0, vec, thr, o_ds, o_ds2, o_e,
                                  o_p);
      tmem_st8(col + kTS, o_ds);
      tmem_st8(col + kTDP, o_ds2);
      tmem_st8(col + kTM, o_e);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[O_EDONE + b]);
    }
    if (ok) ok = wait_w(O_DONE, 0);
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      // a key tile that meets no query tile (none, causal or not) still
      // accumulated at least one quarter: n_q >= 4 always
      store_acc<D>(lane_base, T2::T_A0, p.out0 + orow, key_ok, g, p.scale);
      store_acc<D>(lane_base, T2::T_A1, p.out1 + orow, key_ok, g, 1.f);
    }
  }
  bob_teardown(tmem);
}

template <int D>
cudaError_t launch_bob_bf16_d(const CUtensorMap (&maps)[7], const void* const (&src)[7],
                              const Workspace& ws, float* r_pad, float* g_pad, void* gq, void* gk,
                              void* gv, void* gdo, int BH, int H, int N, bool causal, float scale,
                              uint64_t wait_limit_cycles, int inject_fault, cudaStream_t s) {
  using L = BobLayout<D>;
  static_assert(L::ALLOC <= 232448, "shared memory window exceeds 227 KB");
  for (auto k : {bob_rows_bf16_kernel<D>, bob_cols_bf16_kernel<D>}) {
    const cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
  }
  auto bf = [](const void* x) { return static_cast<const __nv_bfloat16*>(x); };
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
  p.wait_cycles = wait_limit_cycles;
  p.inject_fault = inject_fault;
  const unsigned grid = static_cast<unsigned>(p.T) * static_cast<unsigned>(BH);
  // rows kernel: resident Q, dO, U_Q (src order q, k, v, dout, uq, uk, uv)
  p.res[0] = bf(src[0]);
  p.res[1] = bf(src[3]);
  p.res[2] = bf(src[4]);
  p.res[3] = nullptr;
  p.out0 = static_cast<__nv_bfloat16*>(gq);
  p.out1 = static_cast<__nv_bfloat16*>(gdo);
  bob_rows_bf16_kernel<D><<<grid, kBobThreads, L::ALLOC, s>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // columns kernel: resident K, V, U_K, U_V
  p.res[0] = bf(src[1]);
  p.res[1] = bf(src[2]);
  p.res[2] = bf(src[5]);
  p.res[3] = bf(src[6]);
  p.out0 = static_cast<__nv_bfloat16*>(gk);
  p.out1 = static_cast<__nv_bfloat16*>(gv);
  p.inject_fault = 0;
  bob_cols_bf16_kernel<D><<<grid, kBobThreads, L::ALLOC, s>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bob_bf16(const CUtensorMap (&maps)[7], const void* const (&src)[7],
                            const Workspace& ws, float* r_pad, float* g_pad, void* gq, void* gk,
                            void* gv, void* gdo, int BH, int H, int N, int d, bool causal,
                            float scale, uint64_t wait_limit_cycles, int inject_fault,
                            cudaStream_t s) {
  switch (d) {
    case 32:
      return launch_bob_bf16_d<32>(maps, src, ws, r_pad, g_pad, gq, gk, gv, gdo, BH, H, N, causal,
                                   scale, wait_limit_cycles, inject_fault, s);
    case 64:
      return launch_bob_bf16_d<64>(maps, src, ws, r_pad, g_pad, gq, gk, gv, gdo, BH, H, N, causal,
                                   scale, wait_limit_cycles, inject_fault, s);
    case 128:
      return launch_bob_bf16_d<128>(maps, src, ws, r_pad, g_pad, gq, gk, gv, gdo, BH, H, N,
                                    causal, scale, wait_limit_cycles, inject_fault, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace csa
