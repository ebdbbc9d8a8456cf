// Backward of causal softmax attention on the sm_100a tensor cores (tcgen05).
//
// One CTA per (key tile j of 128 keys, head bh). The CTA keeps K_j and V_j in
// shared memory and walks the query tiles i that can see key tile j (i >= j
// under the causal filter). For each query tile it recomputes the scores
// instead of reading a stored N x N table (ddx issue #243, item 2):
//
//   S^T  = K_j Q_i^T                 (tcgen05 MMA -> TMEM, lanes = keys)
//   P^T  = exp2(S^T * scale*log2e - LSE_i*log2e) -> bf16, back into TMEM
//   dP^T = V_j dO_i^T                (tcgen05 MMA -> TMEM)
//   dS^T = P^T o (dP^T - D_i)        (the max-shift's gradient is dropped,
//                                     ddx issue #243, item 1) -> bf16, into
//                                     TMEM and into shared memory
//   dV_j += P^T dO_i                 (tcgen05, A operand read from TMEM)
//   dK_j += dS^T Q_i                 (tcgen05, A operand read from TMEM;
//                                     accumulators stay in TMEM)
//   dQ_i  = dS K_j                   (tcgen05, A = the shared-memory dS tile
//                                     read transposed -> TMEM -> fp32 red.add)
//
// These are the transposes of ddx PR #162 ("transpose p = w / z per score,
// then p @ v"). Masked (j > i) scores are zeroed in registers on the diagonal
// tile; tiles above the diagonal are never visited.
//
// Warp roles (512 threads, four warpgroups):
//   warps 0-7   two element-wise warpgroups. Thread t of either group owns
//               TMEM lane t (key j0+t); group g handles query columns
//               [64g, 64g+64) of each tile and half of the dK / dV channels
//               in the epilogue. P stays in registers between the P and dS
//               passes.
//   warps 8-11  dQ warpgroup: thread (warp%4)*32 + lane owns query row i0 +
//               that lane; it copies the whole dQ row out of TMEM, releases
//               the columns, then adds the row into the fp32 accumulator with
//               red.global.add while the next tiles are computed.
//   warp 12     MMA issuer (one elected lane); at d = 128 only S^T and dP^T.
//   warp 13     TMA producer (one elected lane): K_j, V_j once; Q_i, dO_i and
//               the tile's LSE / D rows per query tile, three stages deep at
//               d <= 64, two at d = 128.
//   warp 14     d = 128: the second MMA issuer (dV, dK, dQ); idle at d <= 64.
//   warp 15     idle (it completes the fourth warpgroup, which setmaxnreg
//               needs to move registers to the dQ and element-wise warps).
// TMEM (512 columns). d = 128: region A [0,128) holds S^T, then P^T as bf16
// (query q at column 64*(q/64) + (q%64)/2); region B [128,256) holds dP^T,
// then dS^T as bf16 in the same packing; dV [256,384), dK [384,512). dQ takes
// region B after dK has read dS^T. Because P^T and dS^T live in different
// regions, S^T of the next tile only waits for dV and runs while the
// element-wise warps compute dS. d <= 64: two S / P buffers [0,128) and
// [128,256) (query tiles alternate), region B [256,384), dV, dK after it;
// S^T of the next tile is issued into the other buffer before dV of this one,
// and dQ of a tile lands in the first d columns of its own S buffer once dV
// has read P from it, so no MMA of tile i+1 waits for the element-wise warps
// of tile i.
// Every hand-off is an mbarrier; every wait is bounded and reports a timeout.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "tile_walk.cuh"

namespace csa {
namespace {

using namespace sm100;

// Warp roles: two element-wise warpgroups (thread t of group g owns TMEM lane
// t, key row j0 + t, and query columns [QC*g, QC*(g+1))), one dQ warpgroup
// (thread = query row of the dQ tile; a whole row of up to 128 channels), and
// a control warpgroup whose warp MMA_WARP issues the MMAs (at d = 128 it and
// warp MMA2_WARP split them) and warp TMA_WARP the TMA loads. Four
// element-wise warpgroups at
// d <= 64, with dQ read out by them, measured slower (736 vs 791 TFLOP/s on
// 8 heads of 32K tokens): that pass is bound by its MUFU and issue slots, not
// by latency.
template <int D, bool kMask = false>
struct Roles {
  static constexpr int EG = 2;                      // element-wise warpgroups
  static constexpr int QC = 128 / EG;               // query columns per element-wise group
  static constexpr int E_THREADS = 128 * EG;
  static constexpr int DQ_WARP0 = 4 * EG;
  static constexpr int MMA_WARP = DQ_WARP0 + 4;
  static constexpr int TMA_WARP = MMA_WARP + 1;
  // d = 128: a second issuer for the gradient MMAs (dV, dK, dQ), so that they
  // never wait behind a score MMA batch that cannot enter the tensor pipe's
  // queue yet (an MMA issue waits while the queue is full)
  static constexpr int MMA2_WARP = MMA_WARP + 2;
  static constexpr int THREADS = (MMA_WARP + 4) * 32;
  static constexpr int WGS = THREADS / 128;
  // registers a thread holds at launch (the per-block 64K, in steps of 8)
  static constexpr uint32_t LAUNCH_REGS = (65536 / THREADS) / 8 * 8;
  // Budgets after setmaxnreg. One warp of every warpgroup shares an SM
  // sub-partition (16K registers = 512 per lane), and the budgets draw on
  // the registers the block was launched with.
  static constexpr uint32_t R_E = 136;
  // (at d <= 64 a dQ row is half as long, and the control warps' pipelined
  // issue loop and the block-mask walk need the registers it frees)
  static constexpr uint32_t R_DQ = D == 128 ? 144 : 120;
  static constexpr uint32_t R_CTL = D == 128 ? 96 : 120;
  static_assert(EG * R_E + R_DQ + R_CTL <= WGS * LAUNCH_REGS,
                "register split exceeds the launch budget");
  static constexpr int DQ_READERS = 128;            // arrivals on B_DQREAD
  static constexpr int E_CH = D / EG;               // dK / dV channels per group (epilogue)
};
// Pause after each 16-byte dQ reduction of a dQ thread (see the dQ warps).
constexpr unsigned kRedPaceNs = 40;

template <int D>
struct BwdLayout {
  static constexpr int CH = D >= 64 ? 64 : D;   // TMA box width (elements)
  static constexpr int NCH = D / CH;            // boxes per 128-row tile
  static constexpr int ROWB = CH * 2;           // bytes per row inside a box
  static constexpr int CHUNK = kTile * ROWB;    // bytes of one [128][CH] box
  static constexpr int TILE = NCH * CHUNK;      // bytes of one [128][D] bf16 tile
  static constexpr uint32_t SWZ = ROWB == 128 ? kSwizzle128B : kSwizzle64B;
  // At d <= 64 tensor memory holds two S / P buffers, so S of the next query
  // tile is computed while the element-wise warps still work on this one
  // (and dQ of a tile lands in its S buffer once dV has read P); the Q / dO
  // loads then run three stages deep to keep ahead of it.
  static constexpr bool PIPE_S = D <= 64;
  static constexpr int SBUF = PIPE_S ? 2 : 1;
  static constexpr int STAGES = PIPE_S ? 3 : 2;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + TILE;
  static constexpr int Q_OFF = V_OFF + TILE;              // [STAGES] tiles
  static constexpr int DO_OFF = Q_OFF + STAGES * TILE;    // [STAGES] tiles
  static constexpr int DS_OFF = DO_OFF + STAGES * TILE;   // [128 keys][128 queries] bf16
  static constexpr int LSE_OFF = DS_OFF + 32768;          // [STAGES][128] f32
  static constexpr int DV_OFF = LSE_OFF + STAGES * 512;   // [STAGES][128] f32
  static constexpr int BAR_OFF = DV_OFF + STAGES * 512;
  static constexpr int MISC_OFF = BAR_OFF + 32 * 8;
  // block-mask bitmaps of the key tile's column (active tiles, kind-2 tiles):
  // 80 words fill what d = 128 leaves of the window (T <= 2,560 tiles); a
  // longer column is walked in global memory instead
  static constexpr int MASK_WORDS = D == 128 ? 80 : 2048;
  static constexpr int MASK_OFF = MISC_OFF + 64;
  static constexpr int BYTES = MASK_OFF + 2 * 4 * MASK_WORDS;
  // d = 128 fills the 227 KB window, so the window itself must be 1024-byte
  // aligned (checked at run time); smaller d keep 1 KB of alignment slack and
  // at least ~118 KB so that one CTA owns an SM's tensor memory.
  static constexpr bool EXACT = D == 128;
  static constexpr int ALLOC =
      EXACT ? BYTES : ((BYTES + 1024) > 118 * 1024 ? BYTES + 1024 : 118 * 1024);
  // TMEM columns: S / P buffer b at T_S + 128 b; dP / dS; dV; dK. dQ takes
  // region B (dP / dS) at d = 128, after dK has read dS; at d <= 64 the
  // first D columns of its tile's S buffer, after dV has read P.
  static constexpr uint32_t T_S = 0, T_DP = 128 * SBUF, T_DV = T_DP + 128, T_DK = T_DV + D;
  static constexpr bool DQ_OVER_DP = !PIPE_S;
  static constexpr uint32_t T_COLS = 512;
  static_assert(T_DK + D <= T_COLS, "TMEM columns exceeded");
};

// Barrier slots: up to three Q / dO stages, up to two S buffers.
enum Bar {
  B_KV = 0, B_QFULL = 1, B_QEMPTY = 4, B_SFULL = 7, B_DPFULL = 9, B_PFULL, B_DSFULL, B_DVDONE,
  B_DKDONE, B_DQFULL, B_DQREAD = B_DQFULL + 2, B_DONE = B_DQREAD + 2, B_FINAL, B_FINAL2, B_COUNT
};
static_assert(B_COUNT <= 32, "barrier slots");

struct BwdParams {
  const float* lse2;  // [BH][Np], -LSE * log2(e), -inf past N
  const float* dvec;  // [BH][Np], D, 0 past N
  float* dq_acc;      // [BH][T][D/4][128][4]
  __nv_bfloat16* dk;  // rows at qs.row(bh, key), D channels each
  __nv_bfloat16* dv;
  RowStrides ks;      // strides of dk and dv (those of k and v)
  int* status;
  int N, Np, T, BH;   // query rows, rows padded to tiles, query tiles, heads
  int Nk, Tk, q_off;  // keys, key tiles; query row r is position q_off + r
  int G;              // heads per scheduling group (see the CTA order in the kernel)
  int causal;
  const uint8_t* bmask;  // [T][T] tile kinds (0 none, 1 all, 2 key <= query in the tile), or null
  float scale, scale_log2;
  uint64_t wait_cycles;
  int inject_fault;   // 1: never signal the first score tile (tests the timeout path)
};

// Operand descriptors are built once per operand base and stepped by
// constants: a descriptor's start-address field holds address >> 4 in its low
// 14 bits (the shared window lies below 256 KB), so the descriptor of
// base + off is the base's plus off >> 4 for any 16-byte multiple off that
// stays in the window -- one add per MMA operand instead of a mask, a shift
// and an OR on 64-bit values, in the warp that shares its sub-partition with
// two element-wise warps.
//
// K-major operand: rows [128][D] stored as D/CH swizzled boxes; koff steps it
// to the kk-th 16-element K step.
template <int D>
__device__ __forceinline__ uint64_t desc_k0(uint32_t tile) {
  using L = BwdLayout<D>;
  return smem_desc(tile, 16, 8 * L::ROWB, L::SWZ);
}
template <int D>
__host__ __device__ constexpr uint32_t koff(int kk) {
  using L = BwdLayout<D>;
  return static_cast<uint32_t>(((kk * 16) / L::CH) * L::CHUNK + ((kk * 16) % L::CH) * 2) >> 4;
}

// The same [128 rows][D] tile read as an MN-major operand (rows = K,
// columns = M or N); mnoff steps it to the kk-th 16-row K step.
template <int D>
__device__ __forceinline__ uint64_t desc_mn0(uint32_t tile) {
  using L = BwdLayout<D>;
  return smem_desc(tile, L::CHUNK, 8 * L::ROWB, L::SWZ);
}
template <int D>
__host__ __device__ constexpr uint32_t mnoff(int kk) {
  using L = BwdLayout<D>;
  return static_cast<uint32_t>(kk * 16 * L::ROWB) >> 4;
}

// The [128 keys][128 queries] dS tile (two 64-query boxes, 128B swizzle),
// read as the MN-major A operand of dQ = dS K (M = queries, K = keys); its
// kk-th 16-key step lies kk * 2048 bytes on.
__device__ __forceinline__ uint64_t desc_ds0(uint32_t tile) {
  return smem_desc(tile, 16384, 1024, kSwizzle128B);
}

// Byte offset of 16-byte group `g` (8 bf16 columns, 0..15) of row `r` in the
// dS tile.
__device__ __forceinline__ uint32_t ds_offset(int r, int g) {
  return (g >> 3) * 16384 + r * 128 + (((g & 7) ^ (r & 7)) << 4);
}

// TMEM column of the bf16 pair holding query q (q even) of P^T or dS^T
// within its region: each element-wise group packs its QC queries into the
// first QC/2 of its own QC columns.
template <int QC>
__host__ __device__ constexpr uint32_t p_col(int q) { return QC * (q / QC) + (q % QC) / 2; }

// P for this thread's key row over QC queries: p_u = 2^(S_u * scale*log2e -
// LSE_u*log2e), packed as bf16 pairs; the exponent's argument is formed two
// queries at a time by one packed fp32 FMA (fma.rn.f32x2) against the row
// term -LSE*log2e. Queries u < thr are masked (kMasked); off the diagonal
// tile nothing is, and the compare-and-select is skipped.
template <bool kMasked, int QC>
__device__ __forceinline__ void p_from_scores(const uint32_t (&sr)[QC], const float* nlse,
                                              float scale_log2, int thr, uint32_t (&pk)[QC / 2]) {
  const uint64_t c2 = f2(scale_log2, scale_log2);
#pragma unroll
  for (int u = 0; u < QC; u += 4) {
    // one 16-byte broadcast load per four queries: -LSE*log2e as two pairs
    const ulonglong2 l4 = *reinterpret_cast<const ulonglong2*>(nlse + u);
    const float2 x01 = f2_split(fma2(f2(__uint_as_float(sr[u]), __uint_as_float(sr[u + 1])), c2, l4.x));
    const float2 x23 = f2_split(fma2(f2(__uint_as_float(sr[u + 2]), __uint_as_float(sr[u + 3])), c2, l4.y));
    float p0 = ex2_approx(x01.x), p1 = ex2_approx(x01.y);
    float p2 = ex2_approx(x23.x), p3 = ex2_approx(x23.y);
    if (kMasked) {
      if (u < thr) p0 = 0.f;
      if (u + 1 < thr) p1 = 0.f;
      if (u + 2 < thr) p2 = 0.f;
      if (u + 3 < thr) p3 = 0.f;
    }
    pk[u / 2] = pack_bf16x2(p0, p1);
    pk[u / 2 + 1] = pack_bf16x2(p2, p3);
  }
}

template <int D, bool kMask>
__global__ void __launch_bounds__(Roles<D>::THREADS, 1)
    attn_bwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using L = BwdLayout<D>;
  using R = Roles<D, kMask>;
  constexpr int QC = R::QC;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = L::EXACT ? smem_raw
                           : reinterpret_cast<uint8_t*>(
                                 (reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                 ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const volatile int* never = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);  // stays 0
  const float* s_lse = reinterpret_cast<const float*>(smem + L::LSE_OFF);
  const float* s_dv = reinterpret_cast<const float*>(smem + L::DV_OFF);

  const int warp = threadIdx.x >> 5;
  // CTA order: heads in groups of G, the groups one after another; inside a
  // group, key tiles longest-first (key tile 0 has the most query tiles),
  // heads interleaved. The CTAs in flight then touch only a few heads' Q, dO
  // and dQ accumulator, which stay in L2 while every key tile of those heads
  // passes over them; the last group may be smaller.
  const int per_group = p.Tk * p.G;
  const int g0 = (blockIdx.x / per_group) * p.G;
  const int r = blockIdx.x % per_group;
  const int gs = min(p.G, p.BH - g0);
  const int jt = r / gs;
  const int bh = g0 + r % gs;
  const int j0 = jt * kTile;
  // The query tiles this key tile meets, in increasing order: i >= jt under
  // the causal filter, all of them without it, or those a block mask marks.
  // Every role walks them with next_tile, so all agree on tile k of the walk.
  // A block mask's column is read into shared-memory bitmaps once (below)
  // when it fits, else walked byte by byte in global memory.
  uint32_t* s_act = reinterpret_cast<uint32_t*>(smem + L::MASK_OFF);
  uint32_t* s_kind2 = s_act + L::MASK_WORDS;
  const bool mask_bits =
      kMask && (p.T + R::THREADS - 1) / R::THREADS * (R::THREADS / 32) <= L::MASK_WORDS;
  // Queries u of query tile i with u < thr are masked for key row t: keys
  // past N_k mask every query; the causal filter masks queries whose
  // position q_off + 128 i + u is before the key's j0 + t (thr0 = j0 + t -
  // q_off); a block mask's kind-2 tile masks u < t.
  auto tile_thr = [&](int i, int t, int thr0) -> int {
    if constexpr (kMask) {
      if (mask_bits) return bit_set(s_kind2, i) ? t : 0;
      return p.bmask[static_cast<size_t>(i) * p.T + jt] == 2 ? t : 0;
    } else {
      const int th = thr0 - i * kTile;
      return th < 0 ? 0 : th;  // (above 128 every query of the tile is masked)
    }
  };
  auto next_tile = [&](int i) -> int {  // first tile after i that takes part (T if none)
    if constexpr (kMask) {
      if (mask_bits) return next_set_bit(s_act, p.T, i);
      for (++i; i < p.T && p.bmask[static_cast<size_t>(i) * p.T + jt] == 0; ++i) {
      }
      return i;
    } else {
      // under the causal filter the first query tile that sees this key tile:
      // its last row's position q_off + 128 i + 127 must reach key j0
      const int lo = j0 - p.q_off;
      return max(i + 1, (p.causal && lo > kTile - 1) ? lo / kTile : 0);
    }
  };
  int i_first = kMask ? p.T : next_tile(-1);

  // Swizzled operands need a 1024-byte aligned window; nothing has been
  // issued yet, so a misaligned window is reported and every thread returns.
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(p.status, -3);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_KV], 1);
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(&bars[B_QFULL + s], 1);
      mbar_init(&bars[B_QEMPTY + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_DQFULL + s], 1);
      mbar_init(&bars[B_DQREAD + s], R::DQ_READERS);
      mbar_init(&bars[B_SFULL + s], 1);
    }
    mbar_init(&bars[B_DPFULL], 1);
    mbar_init(&bars[B_PFULL], R::E_THREADS);
    mbar_init(&bars[B_DSFULL], R::E_THREADS);
    mbar_init(&bars[B_DVDONE], 1);
    mbar_init(&bars[B_DKDONE], 1);
    mbar_init(&bars[B_DONE], 1);
    mbar_init(&bars[B_FINAL], 1);
    mbar_init(&bars[B_FINAL2], 1);
    *abort_flag = 0;
    *const_cast<volatile int*>(never) = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_base_slot, L::T_COLS);
    tmem_relinquish();
  }
  if constexpr (kMask) {
    if (mask_bits) build_tile_bits<R::THREADS>(p.bmask + jt, p.T, p.T, s_act, s_kind2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  if constexpr (kMask) i_first = next_tile(-1);  // the bitmaps are in place now

  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, kStatusTimeout);
  };

  // Registers move from the control warpgroup to the others; each budget is
  // set at the head of its role's branch so that the compiler allocates that
  // branch's code against it.
  if (warp >= R::MMA_WARP) {
    regs_to<R::R_CTL, R::LAUNCH_REGS>();
  if (warp == R::TMA_WARP) {
    // ------------------------------------------------ TMA producer
    if (elect_one_sync()) {
      const int hh = bh % p.ks.H, hb = bh / p.ks.H;  // head and batch: TMA coordinates
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_do);
      mbar_arrive_expect_tx(&bars[B_KV], 2 * L::TILE);
      for (int c = 0; c < L::NCH; ++c) {
        tma_load_4d(smem + L::K_OFF + c * L::CHUNK, &tm_k, &bars[B_KV], c * L::CH, j0, hh, hb);
        tma_load_4d(smem + L::V_OFF + c * L::CHUNK, &tm_v, &bars[B_KV], c * L::CH, j0, hh, hb);
      }
      bool ok = true;
      int issued = 0;
      for (int it = 0, i = i_first; i < p.T; ++it, i = next_tile(i)) {
        const int s = it % L::STAGES;
        if (it >= L::STAGES &&
            !(ok = mbar_wait(&bars[B_QEMPTY + s], ((it - L::STAGES) / L::STAGES) & 1, p.wait_cycles,
                             abort_flag)))
          break;
        // (a debug build redirects an out-of-range tile to tile 0)
        const int i0 =
            (CSA_IN_BOUNDS(i >= 0 && i < p.T && jt < p.Tk && bh < p.BH, p.status) ? i : 0) * kTile;
        uint64_t* bar = &bars[B_QFULL + s];
        mbar_arrive_expect_tx(bar, 2 * L::TILE + 2 * 512);
        for (int c = 0; c < L::NCH; ++c) {
          tma_load_4d(smem + L::Q_OFF + s * L::TILE + c * L::CHUNK, &tm_q, bar, c * L::CH, i0,
                      hh, hb);
          tma_load_4d(smem + L::DO_OFF + s * L::TILE + c * L::CHUNK, &tm_do, bar, c * L::CH,
                      i0, hh, hb);
        }
        bulk_load(smem + L::LSE_OFF + s * 512, p.lse2 + static_cast<size_t>(bh) * p.Np + i0, 512,
                  bar);
        bulk_load(smem + L::DV_OFF + s * 512, p.dvec + static_cast<size_t>(bh) * p.Np + i0, 512,
                  bar);
        ++issued;
      }
      if (!ok) fail();
      // Every load issued has landed before the CTA can exit (bounded).
      mbar_wait(&bars[B_KV], 0, p.wait_cycles, never);
      for (int w = issued > L::STAGES ? issued - L::STAGES : 0; w < issued; ++w)
        mbar_wait(&bars[B_QFULL + w % L::STAGES], (w / L::STAGES) & 1, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp == R::MMA_WARP || (!L::PIPE_S && warp == R::MMA2_WARP)) {
    // ------------------------------------------------ MMA issuers
    // Each wait guards one TMEM or shared-memory region against the MMA that
    // overwrites it. d = 128, two issuers: warp MMA_WARP issues the score
    // MMAs S(i+1) (it overwrites P(i), so it waits for dV(i)) and dP(i+1) (it
    // overwrites region B, where dQ(i) lands, so it waits for dQ(i)'s
    // read-out), with S(0) and dP(0) before the loop; warp MMA2_WARP issues
    // dV(i), dK(i) and dQ(i) (which overwrites dS^T(i), so it waits for
    // dK(i)). Every barrier is committed by one thread, and each issuer's
    // queue no longer holds the other's MMAs behind a full tensor pipe.
    // d <= 64 (two S buffers), one issuer: S(i+1), dV(i), dK(i), dQ(i),
    // dP(i+1): S(i+1) goes into the other buffer as soon as its last reader
    // (the read-out of dQ(i-1)) is done, so the element-wise warps find it
    // ready when they finish dS(i).
    if (elect_one_sync()) {
      const uint32_t sK = sbase + L::K_OFF, sV = sbase + L::V_OFF, sdS = sbase + L::DS_OFF;
      constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t ID_KV = idesc_bf16(128, D, false, true);
      constexpr uint32_t ID_Q = idesc_bf16(128, D, true, true);
      auto wait = [&](int b, uint32_t parity) {
        return mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag);
      };
      auto stage_q = [&](int it) { return sbase + L::Q_OFF + (it % L::STAGES) * L::TILE; };
      auto stage_do = [&](int it) { return sbase + L::DO_OFF + (it % L::STAGES) * L::TILE; };
      auto qfull = [&](int it) { return wait(B_QFULL + it % L::STAGES, (it / L::STAGES) & 1); };
      auto sbuf = [&](int it) { return L::T_S + 128 * (it % L::SBUF); };
      // S^T(it) = K_j Q_i^T -> S buffer it % SBUF
      const uint64_t dK = desc_k0<D>(sK), dV = desc_k0<D>(sV);
      const uint64_t dKmn = desc_mn0<D>(sK), dDS = desc_ds0(sdS);
      auto issue_s = [&](int it) {
        const uint64_t dQ = desc_k0<D>(stage_q(it));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + sbuf(it), dK + koff<D>(kk), dQ + koff<D>(kk), ID_S, kk > 0);
        if (!(p.inject_fault && it == 0)) mma_commit(&bars[B_SFULL + it % L::SBUF]);
      };
      // dP^T(it) = V_j dO_i^T -> region B
      auto issue_dp = [&](int it) {
        const uint64_t ddO = desc_k0<D>(stage_do(it));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + L::T_DP, dV + koff<D>(kk), ddO + koff<D>(kk), ID_S, kk > 0);
        mma_commit(&bars[B_DPFULL]);
      };
      // dV_j += P^T dO_i, P^T read from the tile's S buffer (K = 128 queries)
      auto issue_dv = [&](int it) {
        const uint64_t ddO = desc_mn0<D>(stage_do(it));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + L::T_DV, tmem + sbuf(it) + p_col<QC>(16 * kk), ddO + mnoff<D>(kk), ID_KV,
                 (it > 0 || kk > 0));
        mma_commit(&bars[B_DVDONE]);
      };
      // dK_j += dS^T Q_i, dS^T read from region B. dK(it) is the last reader
      // of Q_i / dO_i's stage: S^T(it) and dP^T(it) completed before their
      // results could be consumed, dV(it) was issued before it by the same
      // thread (or, at d = 128, by the same second issuer), and the
      // element-wise warps' LSE / D reads ended before dS^T(it) was signalled;
      // dQ(it) reads only dS and the resident K. So the stage is released
      // here, an MMA chain earlier than after dQ(it).
      auto issue_dk = [&](int it) {
        const uint64_t dQ = desc_mn0<D>(stage_q(it));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + L::T_DK, tmem + L::T_DP + p_col<QC>(16 * kk), dQ + mnoff<D>(kk), ID_KV,
                 (it > 0 || kk > 0));
        mma_commit(&bars[B_DKDONE]);
        mma_commit(&bars[B_QEMPTY + it % L::STAGES]);
      };
      // dQ_i = dS K_j (dS from shared memory) -> region B (d = 128) or the
      // tile's S buffer (d <= 64)
      auto issue_dq = [&](int it) {
        const uint32_t dst = L::DQ_OVER_DP ? L::T_DP : sbuf(it);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + dst, dDS + kk * 128, dKmn + mnoff<D>(kk), ID_Q, kk > 0);
        mma_commit(&bars[B_DQFULL + (it & 1)]);
      };
      const bool scores = L::PIPE_S || warp == R::MMA_WARP;  // S and dP
      const bool grads = L::PIPE_S || warp == R::MMA2_WARP;  // dV, dK, dQ
      bool ok = true;
      if (scores && i_first < p.T && (ok = wait(B_KV, 0) && qfull(0))) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      if (!scores && i_first < p.T) ok = wait(B_KV, 0);
      for (int it = 0, i = i_first; ok && i < p.T; ++it, i = next_tile(i)) {
        const bool more = next_tile(i) < p.T;
        if constexpr (L::PIPE_S) {
          if (more) {
            // S(it+1) reuses the buffer of tile it-1, free once dQ(it-1) is read out
            if (!(ok = qfull(it + 1))) break;
            if (it >= 1 && !(ok = wait(B_DQREAD + ((it - 1) & 1), ((it - 1) >> 1) & 1))) break;
            tc_fence_after();
            issue_s(it + 1);
          }
          if (!(ok = wait(B_PFULL, it & 1))) break;
          tc_fence_after();
          issue_dv(it);
          if (!(ok = wait(B_DSFULL, it & 1))) break;
          tc_fence_after();
          issue_dk(it);
          // dQ(it) overwrites P(it), which dV(it) reads
          if (!(ok = wait(B_DVDONE, it & 1))) break;
          tc_fence_after();
          issue_dq(it);
          if (more) {
            // dP(it+1) overwrites dS^T(it), which dK(it) reads
            if (!(ok = wait(B_DKDONE, it & 1))) break;
            tc_fence_after();
            issue_dp(it + 1);
          }
        } else if (scores) {
          if (more) {
            // S^T(it+1) overwrites P^T(it), which dV(it) reads.
            if (!(ok = qfull(it + 1))) break;
            if (!(ok = wait(B_DVDONE, it & 1))) break;
            tc_fence_after();
            issue_s(it + 1);
            // dP^T(it+1) overwrites region B, where dQ(it) lands; its
            // read-out also means dQ(it) has finished reading dS(it) from
            // shared memory, which the element-wise warps overwrite next
            if (!(ok = wait(B_DQREAD + (it & 1), (it >> 1) & 1))) break;
            tc_fence_after();
            issue_dp(it + 1);
          }
        } else {
          if (!(ok = wait(B_PFULL, it & 1))) break;
          tc_fence_after();
          issue_dv(it);
          if (!(ok = wait(B_DSFULL, it & 1))) break;
          tc_fence_after();
          issue_dk(it);
          if (!(ok = wait(B_DKDONE, it & 1))) break;  // dQ(it) overwrites dS^T(it)
          tc_fence_after();
          issue_dq(it);
        }
      }
      if (!ok) {
        fail();
      } else if (grads) {
        mma_commit(&bars[B_DONE]);
      }
      // Every MMA this thread issued has finished before TMEM is freed.
      const int fin = warp == R::MMA_WARP ? B_FINAL : B_FINAL2;
      mma_commit(&bars[fin]);
      mbar_wait(&bars[fin], 0, p.wait_cycles, never);
    }
    __syncwarp();
  }
  } else if (warp >= R::DQ_WARP0) {
    regs_to<R::R_DQ, R::LAUNCH_REGS>();
    // ------------------------------------------------ dQ warpgroup
    const int t = ((warp & 3) << 5) | (threadIdx.x & 31);  // TMEM lane = query row
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    auto wait_w = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag));
    };
    bool ok = true;
    for (int it = 0, i = i_first; i < p.T; ++it, i = next_tile(i)) {
      const int b = it & 1;
      if (!(ok = wait_w(B_DQFULL + b, (it >> 1) & 1))) break;
      tc_fence_after();
      // The whole row first, so the columns are released before the atomics.
      uint32_t r[D];
#pragma unroll
      for (int c = 0; c < D; c += 32)
        tmem_ld32(lane_base + (L::DQ_OVER_DP ? L::T_DP : L::T_S + 128 * (it % L::SBUF)) + c,
                  *reinterpret_cast<uint32_t(*)[32]>(r + c));
      tmem_ld_wait(r);
      tc_fence_before();
      mbar_arrive(&bars[B_DQREAD + b]);
      if (i * kTile + t < p.N &&  // a query row of this head
          CSA_IN_BOUNDS(i >= 0 && i < p.T && bh < p.BH && t < kTile, p.status)) {
        float* acc = p.dq_acc + (static_cast<size_t>(bh) * p.T + i) * (D / 4) * 512 + t * 4;
        // Metered: a burst of reductions fills the sub-partition's memory
        // instruction queue, and the element-wise warps' TMEM and shared-memory
        // accesses then wait behind it. Spaced out, the reductions of one tile
        // drain during the next tile's work.
#pragma unroll
        for (int v = 0; v < D / 4; ++v) {
          red_add_v4(acc + v * 512, __uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                     __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          __nanosleep(kRedPaceNs);
        }
      }
    }
    if (!ok) fail();
  } else {
    regs_to<R::R_E, R::LAUNCH_REGS>();
    // ------------------------------------------------ element-wise warpgroups
    const int t = threadIdx.x & 127;  // TMEM lane: key row
    const int g = threadIdx.x >> 7;   // query columns [QC*g, QC*(g+1)), channels [g*E_CH, ...)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = j0 + t;
    const int qb = QC * g;
    // causal threshold of this key row at query tile 0 (none without the filter)
    const int thr0 = p.causal ? key - p.q_off : -(1 << 30);
    // Outcome of a wait, made uniform across the warp: the TMEM accesses that
    // follow are warp-collective, so a warp must never split on a timeout.
    auto wait_w = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag));
    };
    bool ok = true;
    int it = 0;
    for (int i = i_first; i < p.T; ++it, i = next_tile(i)) {
      const int s = it % L::STAGES;
      // LSE_i, D_i in shared memory
      if (!(ok = wait_w(B_QFULL + s, (it / L::STAGES) & 1))) break;
      const float* lse_s = s_lse + s * 128;
      const float* d_s = s_dv + s * 128;
      // queries with local index < thr are masked for this key row (kind 2:
      // the key must not lie after the query inside the tile)
      const int thr = key >= p.Nk ? kTile : tile_thr(i, t, thr0);

      // ---- P^T = exp2(S^T * scale*log2e - LSE*log2e) -> bf16 into region A
      const uint32_t t_s = L::T_S + 128 * (it % L::SBUF);  // this tile's S / P buffer
      if (!(ok = wait_w(B_SFULL + it % L::SBUF, (it / L::SBUF) & 1))) break;
      tc_fence_after();
      uint32_t pk[QC / 2];  // this thread's QC P values as bf16 pairs, kept for the dS pass
      {
        uint32_t sr[QC];
        tmem_ld<QC>(lane_base + t_s + qb, sr);
        tmem_ld_wait(sr);
        // Only the diagonal tile and the key tile past N mask anything.
        if (__any_sync(0xffffffffu, thr > qb))
          p_from_scores<true, QC>(sr, lse_s + qb, p.scale_log2, thr - qb, pk);
        else
          p_from_scores<false, QC>(sr, lse_s + qb, p.scale_log2, 0, pk);
      }
      // all of this group's S^T columns were read above, so the packed P may
      // overwrite the first half of them
#pragma unroll
      for (int c = 0; c < QC / 2; c += 16)
        tmem_st16(lane_base + t_s + p_col<QC>(qb) + c,
                  *reinterpret_cast<uint32_t(*)[16]>(pk + c));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL]);

      // ---- dS^T = P^T o (dP^T - D) -> bf16 into region B and shared memory
      if (!(ok = wait_w(B_DPFULL, it & 1))) break;
      tc_fence_after();
      uint32_t dk[QC / 2];
      {
        uint32_t dr[QC];
        tmem_ld<QC>(lane_base + L::T_DP + qb, dr);
        tmem_ld_wait(dr);
#pragma unroll
        for (int u = 0; u < QC; u += 4) {
          const int q0 = qb + u;
          const ulonglong2 d4 = *reinterpret_cast<const ulonglong2*>(d_s + q0);
          const float2 pa = unpack_bf16x2(pk[u / 2]);
          const float2 pb = unpack_bf16x2(pk[u / 2 + 1]);
          const float2 x01 = f2_split(mul2(f2(pa.x, pa.y),
              sub2(f2(__uint_as_float(dr[u]), __uint_as_float(dr[u + 1])), d4.x)));
          const float2 x23 = f2_split(mul2(f2(pb.x, pb.y),
              sub2(f2(__uint_as_float(dr[u + 2]), __uint_as_float(dr[u + 3])), d4.y)));
          dk[u / 2] = pack_bf16x2(x01.x, x01.y);
          dk[u / 2 + 1] = pack_bf16x2(x23.x, x23.y);
        }
      }
      // dS^T for dK (TMEM A operand); all dP^T columns of the group were read above
#pragma unroll
      for (int c = 0; c < QC / 2; c += 16)
        tmem_st16(lane_base + L::T_DP + p_col<QC>(qb) + c,
                  *reinterpret_cast<uint32_t(*)[16]>(dk + c));
      // dS for dQ (shared memory, read transposed by the MMA). dQ(it-1) has
      // finished reading the previous tile: dP^T(it) was issued after it.
      uint8_t* sdS = smem + L::DS_OFF;
#pragma unroll
      for (int v = 0; v < QC / 8; ++v)
        st_shared_v4(smem_u32(sdS) + ds_offset(t, qb / 8 + v), dk[4 * v], dk[4 * v + 1],
                     dk[4 * v + 2], dk[4 * v + 3]);
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_DSFULL]);
    }
    if (ok) ok = wait_w(B_DONE, 0);
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      // Epilogue: dV_j and scale * dK_j rows -> bf16, group g writing channels
      // [g*E_CH, (g+1)*E_CH). All lanes load; only the stores are predicated.
      const bool key_ok = key < p.Nk;
      __nv_bfloat16* dv_row = p.dv + p.ks.row(bh, key_ok ? key : 0);
      __nv_bfloat16* dk_row = p.dk + p.ks.row(bh, key_ok ? key : 0);
      constexpr int W = R::E_CH >= 32 ? 32 : R::E_CH;
      const bool any = it > 0;  // a key tile that meets no query tile has dK = dV = 0
#pragma unroll 1
      for (int c = 0; c < R::E_CH / W; ++c) {
        const int ch = g * R::E_CH + W * c;
        uint32_t rv[W], rk[W];
        if (any) {
          tmem_ld<W>(lane_base + L::T_DV + ch, rv);
          tmem_ld<W>(lane_base + L::T_DK + ch, rk);
          tmem_ld_wait(rv, rk);
        } else {
#pragma unroll
          for (int u = 0; u < W; ++u) rv[u] = rk[u] = 0u;
        }
        const bool store_ok = key_ok && CSA_IN_BOUNDS(bh < p.BH && ch + W <= D, p.status);
#pragma unroll
        for (int v = 0; v < W / 8 && store_ok; ++v) {
          uint4 ov, ok4;
          ov.x = pack_bf16x2(__uint_as_float(rv[8 * v + 0]), __uint_as_float(rv[8 * v + 1]));
          ov.y = pack_bf16x2(__uint_as_float(rv[8 * v + 2]), __uint_as_float(rv[8 * v + 3]));
          ov.z = pack_bf16x2(__uint_as_float(rv[8 * v + 4]), __uint_as_float(rv[8 * v + 5]));
          ov.w = pack_bf16x2(__uint_as_float(rv[8 * v + 6]), __uint_as_float(rv[8 * v + 7]));
          ok4.x = pack_bf16x2(p.scale * __uint_as_float(rk[8 * v + 0]),
                              p.scale * __uint_as_float(rk[8 * v + 1]));
          ok4.y = pack_bf16x2(p.scale * __uint_as_float(rk[8 * v + 2]),
                              p.scale * __uint_as_float(rk[8 * v + 3]));
          ok4.z = pack_bf16x2(p.scale * __uint_as_float(rk[8 * v + 4]),
                              p.scale * __uint_as_float(rk[8 * v + 5]));
          ok4.w = pack_bf16x2(p.scale * __uint_as_float(rk[8 * v + 6]),
                              p.scale * __uint_as_float(rk[8 * v + 7]));
          *reinterpret_cast<uint4*>(dv_row + ch + 8 * v) = ov;
          *reinterpret_cast<uint4*>(dk_row + ch + 8 * v) = ok4;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::T_COLS);
  }
}

template <int D>
cudaError_t launch_bwd_bf16_d(const TmaMaps& m, const Workspace& ws, void* dk, void* dv, int BH,
                              const Extent& ex, bool causal, float scale, uint64_t wait_cycles,
                              int inject, const uint8_t* bmask, const RowStrides& ks,
                              cudaStream_t s) {
  using L = BwdLayout<D>;
  static_assert(L::ALLOC <= 232448, "shared memory window exceeds 227 KB");
  auto kern = bmask ? attn_bwd_bf16_sm100_kernel<D, true> : attn_bwd_bf16_sm100_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  // The setmaxnreg split redistributes exactly the registers the block is
  // launched with; with fewer at launch the increases could never be served.
  static const cudaError_t regs_ok = []() {
    for (auto k : {attn_bwd_bf16_sm100_kernel<D, false>, attn_bwd_bf16_sm100_kernel<D, true>}) {
      cudaFuncAttributes fa;
      const cudaError_t r = cudaFuncGetAttributes(&fa, k);
      if (r != cudaSuccess) return r;
      if (fa.numRegs != static_cast<int>(Roles<D>::LAUNCH_REGS)) return cudaErrorInvalidConfiguration;
    }
    return cudaSuccess;
  }();
  if (regs_ok != cudaSuccess) return regs_ok;
  BwdParams p;
  p.lse2 = ws.lse_pad;
  p.dvec = ws.d_pad;
  p.dq_acc = ws.dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.status = ws.status;
  p.N = ex.nq;
  p.Np = ws.Np;
  p.T = ws.Np / kTile;
  p.BH = BH;
  p.Nk = ex.nk;
  p.Tk = (ex.nk + kTile - 1) / kTile;
  p.q_off = ex.q_off;
  // Heads per group: as many as fit, with their Q and dO tiles (bf16) and dQ
  // accumulator (fp32), in about a third of L2.
  int dev = 0, l2 = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0)
    l2 = 126 << 20;
  const size_t head_bytes = static_cast<size_t>(ws.Np) * D * 8;
  p.G = static_cast<int>(std::max<size_t>(1, std::min<size_t>(BH, (l2 / 3) / head_bytes)));
  p.causal = causal ? 1 : 0;
  p.bmask = bmask;
  p.ks = ks;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_cycles = wait_cycles;
  p.inject_fault = inject;
  const unsigned grid = static_cast<unsigned>(p.Tk) * static_cast<unsigned>(BH);
  kern<<<grid, Roles<D>::THREADS, L::ALLOC, s>>>(m.a, m.b, m.c, m.d, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_bf16(const TmaMaps& maps, const Workspace& ws, void* dk, void* dv, int BH,
                            const Extent& ex, int d, bool causal, float scale,
                            uint64_t wait_limit_cycles, int inject_fault,
                            const uint8_t* block_mask, const RowStrides& ks, cudaStream_t s) {
  switch (d) {
    case 32:
      return launch_bwd_bf16_d<32>(maps, ws, dk, dv, BH, ex, causal, scale, wait_limit_cycles,
                                   inject_fault, block_mask, ks, s);
    case 64:
      return launch_bwd_bf16_d<64>(maps, ws, dk, dv, BH, ex, causal, scale, wait_limit_cycles,
                                   inject_fault, block_mask, ks, s);
    case 128:
      return launch_bwd_bf16_d<128>(maps, ws, dk, dv, BH, ex, causal, scale, wait_limit_cycles,
                                    inject_fault, block_mask, ks, s);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace csa
