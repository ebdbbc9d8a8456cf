// Forward of causal softmax attention on the sm_100a tensor cores (tcgen05).
//
// One CTA per (query tile i of 128 rows, head bh), walking the key tiles j
// that the causal filter lets tile i see (j <= i):
//
//   S_j = Q_i K_j^T                    (tcgen05 MMA -> TMEM, lane = query row)
//   m   = running row maximum of S * scale*log2e
//   P_j = exp2(S_j * scale*log2e - m)  -> bf16, in place in S_j's columns
//   O  += P_j V_j                      (tcgen05, A = P_j read from TMEM; O
//                                       accumulates in TMEM across tiles)
//   z  += rowsum P_j
//
// and writes O / z (bf16) and LSE = (m + log2 z) ln 2, the one saved number
// per row of ddx issue #243 (item 2). The max-shifted softmax is the
// `weights` / `norm` steps of ddx issue #217's repro; the key filter is its
// `WHERE q.pos >= k.pos` (diagonal kept). m is only raised when the row
// maximum exceeds it by more than 8 (P stays below 2^8, exact in fp32 and
// well inside bf16's range); O and z are then scaled by 2^(m_old - m_new)
// before the next P V accumulates, which after the first tiles is rare.
//
// Warps (384 threads): 0-7 two softmax warpgroups (thread t of group g owns
// query row i0 + t = TMEM lane t and key columns [64g, 64g+64) of every S
// tile). Each group keeps its own running maximum m_g, sum z_g and
// accumulator O_g = sum over its keys of P V (the P V MMA runs as two K = 64
// halves), so the groups never wait for each other inside the key loop; the
// epilogue combines the halves once:
//   M = max(m_0, m_1), a_g = 2^(m_g - M), O = (a_0 O_0 + a_1 O_1) / (a_0 z_0 + a_1 z_1).
// Warp 8 issues the MMAs, warp 9 loads K tiles and warp 10 V tiles by TMA;
// warp 11 idles. TMEM: S buffers from column 0 (three at d <= 64, two at
// d = 128), then O_0 and O_1: S_{j+1} (and at d <= 64 S_{j+2}) is computed
// while the softmax works on S_j and P_{j-1} V_{j-1} accumulates.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "tile_walk.cuh"

namespace csa {

__device__ int g_fwd_status;  // forward's status word (per device)

int* fwd_status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fwd_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

namespace {

using namespace sm100;

constexpr int kFwdThreads = 384;
constexpr int kSoftmaxThreads = 256;  // warps 0-7
constexpr int kFwdMmaWarp = 8;
constexpr int kFwdKWarp = 9;
constexpr int kFwdVWarp = 10;
constexpr float kRescaleMargin = 8.f;  // log2 units: m is raised when the max exceeds it by this

template <int D>
struct FwdLayout {
  static constexpr int CH = D >= 64 ? 64 : D;
  static constexpr int NCH = D / CH;
  static constexpr int ROWB = CH * 2;
  static constexpr int CHUNK = kTile * ROWB;
  static constexpr int TILE = NCH * CHUNK;
  static constexpr uint32_t SWZ = ROWB == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;        // [2] tiles
  static constexpr int V_OFF = K_OFF + 2 * TILE;    // [2] tiles
  static constexpr int XM_OFF = V_OFF + 2 * TILE;   // [2][2][128] f32: the groups' maxima, sums
  static constexpr int BAR_OFF = XM_OFF + 2048;
  static constexpr int MISC_OFF = BAR_OFF + 32 * 8;
  // block-mask bitmaps of the query tile's row (active tiles, kind-2 tiles),
  // T <= 65,280 tiles; a longer row is walked in global memory instead
  static constexpr int MASK_WORDS = 2040;
  static constexpr int MASK_OFF = MISC_OFF + 64;
  static constexpr int BYTES = MASK_OFF + 2 * 4 * MASK_WORDS;
  static constexpr int ALLOC = (BYTES + 1024) > 118 * 1024 ? (BYTES + 1024) : 118 * 1024;
  // S buffers in TMEM, then one O accumulator per softmax group (O_g at
  // T_O + g * D); at d = 128 the accumulators leave room for two S buffers
  static constexpr int SBUF = D == 128 ? 2 : 3;
  static constexpr uint32_t T_S = 0, T_O = 128 * SBUF;
  static constexpr uint32_t T_COLS = 512;
  static constexpr int HALF_D = D / 2;              // O channels each group writes out
  static_assert(T_O + 2 * D <= T_COLS, "TMEM columns exceeded");
};

// F_PFULL + 2g + (j & 1): group g's half of P_j is in TMEM. A group can
// finish two tiles before the issuer looks (the other group holding the
// issuer up) without the phases aliasing: its P_{j+2} needs S_{j+2}, issued
// only after P_j was consumed. F_PVDONE + (j & 1): group 0's half of
// P_j V_j has completed, F_PVDONE1 + (j & 1): both halves have. F_XCHG: the
// epilogue's exchange of the groups' maxima and sums.
enum FBar {
  F_Q = 0, F_KFULL = 1, F_KEMPTY = 3, F_VFULL = 5, F_VEMPTY = 7, F_SFULL = 9,
  F_PFULL = F_SFULL + 3, F_PVDONE = F_PFULL + 4, F_PVDONE1 = F_PVDONE + 2, F_XCHG = F_PVDONE1 + 2,
  F_FINAL, F_COUNT
};
static_assert(F_COUNT <= 32, "barrier slots");

struct FwdParams {
  __nv_bfloat16* o;  // rows at os.row(bh, i), D channels each
  RowStrides os;     // strides of o
  float* lse;        // [BH][N]
  int* status;
  int N, T, BH;      // query rows, query tiles, heads
  int Nk, Tk, q_off; // keys, key tiles; query row r is position q_off + r
  int G;             // heads per scheduling group (see the CTA order)
  int causal;
  const uint8_t* bmask;  // [T][T] tile kinds (0 none, 1 all, 2 key <= query in the tile), or null
  float scale_log2;
  uint64_t wait_cycles;
};

template <int D>
__device__ __forceinline__ uint64_t fdesc_kmajor(uint32_t tile, int kk) {
  using L = FwdLayout<D>;
  const int e = kk * 16;
  return smem_desc(tile + (e / L::CH) * L::CHUNK + (e % L::CH) * 2, 16, 8 * L::ROWB, L::SWZ);
}
template <int D>
__device__ __forceinline__ uint64_t fdesc_mnmajor(uint32_t tile, int kk) {
  using L = FwdLayout<D>;
  return smem_desc(tile + kk * 16 * L::ROWB, L::CHUNK, 8 * L::ROWB, L::SWZ);
}
// TMEM column of the bf16 pair holding key k (k even) of P_j in its S buffer:
// each softmax group packs its 64 keys into the first 32 of its own columns.
__host__ __device__ constexpr uint32_t fp_col(int k) { return 64 * (k >> 6) + ((k & 63) >> 1); }

template <int D, bool kMask>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const volatile int* never = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);
  float* xm = reinterpret_cast<float*>(smem + L::XM_OFF);  // [m, z][2 groups][128 rows]

  const int warp = threadIdx.x >> 5;
  // CTA order: heads in groups of G (their K and V stay in L2 while all of
  // their query tiles pass), longest query tile first inside a group.
  const int per_group = p.T * p.G;
  const int g0 = (blockIdx.x / per_group) * p.G;
  const int r = blockIdx.x % per_group;
  const int gs = min(p.G, p.BH - g0);
  // (a block mask is taken to be causal-like: later query tiles first too)
  const int it_q = (p.causal || kMask) ? p.T - 1 - r / gs : r / gs;
  const int bh = g0 + r % gs;
  const int hh = bh % p.os.H, hb = bh / p.os.H;  // head and batch: TMA coordinates
  const int i0 = it_q * kTile;
  // The key tiles this query tile meets, in increasing order: j <= i under
  // the causal filter, all of them without it, or those a block mask marks.
  // Every role walks them with next_tile, so all agree on tile k of the walk.
  // A block mask's row is read into shared-memory bitmaps once (below) when
  // it fits, else walked byte by byte in global memory.
  uint32_t* s_act = reinterpret_cast<uint32_t*>(smem + L::MASK_OFF);
  uint32_t* s_kind2 = s_act + L::MASK_WORDS;
  const uint8_t* mask_row = kMask ? p.bmask + static_cast<size_t>(it_q) * p.T : nullptr;
  const bool mask_bits =
      kMask && (p.T + kFwdThreads - 1) / kFwdThreads * (kFwdThreads / 32) <= L::MASK_WORDS;
  auto tile_kind = [&](int j) -> int {
    if constexpr (kMask) {
      if (mask_bits) return bit_set(s_kind2, j) ? 2 : 1;
      return mask_row[j];
    } else {
      return !p.causal ? 1 : (j < it_q ? 1 : (j == it_q ? 2 : 0));
    }
  };
  // last key tile the causal filter lets this query tile see (key position
  // <= q_off + its last row's index)
  const int j_last = min(p.Tk - 1, (p.q_off + i0 + kTile - 1) / kTile);
  auto next_tile = [&](int j) -> int {  // first tile after j that takes part (Tk if none)
    if constexpr (kMask) {
      if (mask_bits) return next_set_bit(s_act, p.Tk, j);
      for (++j; j < p.Tk && mask_row[j] == 0; ++j) {
      }
      return j;
    } else {
      return (p.causal && j + 1 > j_last) ? p.Tk : j + 1;
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars[F_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[F_KFULL + s], 1);
      mbar_init(&bars[F_KEMPTY + s], 1);
      mbar_init(&bars[F_VFULL + s], 1);
      mbar_init(&bars[F_VEMPTY + s], 1);
      mbar_init(&bars[F_PVDONE + s], 1);
      mbar_init(&bars[F_PVDONE1 + s], 1);
    }
    for (int s = 0; s < 4; ++s) mbar_init(&bars[F_PFULL + s], kSoftmaxThreads / 2);
    for (int s = 0; s < 3; ++s) mbar_init(&bars[F_SFULL + s], 1);
    mbar_init(&bars[F_XCHG], kSoftmaxThreads);
    mbar_init(&bars[F_FINAL], 1);
    *abort_flag = 0;
    *const_cast<volatile int*>(never) = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_base_slot, L::T_COLS);
    tmem_relinquish();
  }
  if constexpr (kMask) {
    if (mask_bits) build_tile_bits<kFwdThreads>(mask_row, 1, p.T, s_act, s_kind2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int j_first = next_tile(-1);
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, kStatusTimeout);
  };

  if (warp == kFwdKWarp || warp == kFwdVWarp) {
    // ------------------------------------------------ TMA: Q and K (warp 9), V (warp 10)
    if (elect_one_sync()) {
      const bool is_k = warp == kFwdKWarp;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      const int full = is_k ? F_KFULL : F_VFULL, empty = is_k ? F_KEMPTY : F_VEMPTY;
      const int off = is_k ? L::K_OFF : L::V_OFF;
      prefetch_tensormap(map);
      if (is_k) {
        prefetch_tensormap(&tm_q);
        mbar_arrive_expect_tx(&bars[F_Q], L::TILE);
        for (int c = 0; c < L::NCH; ++c)
          tma_load_4d(smem + L::Q_OFF + c * L::CHUNK, &tm_q, &bars[F_Q], c * L::CH, i0, hh, hb);
      }
      bool ok = true;
      int issued = 0;
      for (int jt = 0, j = j_first; j < p.Tk; ++jt, j = next_tile(j)) {
        const int s = jt & 1;
        // K_j is free once S_j has been computed, V_j once P_j V_j has.
        if (jt >= 2 &&
            !(ok = mbar_wait(&bars[empty + s], ((jt - 2) >> 1) & 1, p.wait_cycles, abort_flag)))
          break;
        mbar_arrive_expect_tx(&bars[full + s], L::TILE);
        // (a debug build redirects an out-of-range tile to tile 0)
        const int j_ld = CSA_IN_BOUNDS(j >= 0 && j < p.Tk && bh < p.BH, p.status) ? j : 0;
        for (int c = 0; c < L::NCH; ++c)
          tma_load_4d(smem + off + s * L::TILE + c * L::CHUNK, map, &bars[full + s], c * L::CH,
                      j_ld * kTile, hh, hb);
        ++issued;
      }
      if (!ok) fail();
      // Every load issued has landed before the CTA can exit (bounded).
      if (is_k) mbar_wait(&bars[F_Q], 0, p.wait_cycles, never);
      for (int w = issued > 2 ? issued - 2 : 0; w < issued; ++w)
        mbar_wait(&bars[full + (w & 1)], (w >> 1) & 1, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp == kFwdMmaWarp) {
    // ------------------------------------------------ MMA issuer
    // Order: S_0, S_1, then per key tile j: the two halves of P_j V_j, then
    // S_{j+2} into the buffer P_{j+2-SBUF} occupied, once that tile's P V has
    // completed (P_{j-1} with three buffers: never a pipe drain, because P_j
    // V_j is already queued; P_j with two).
    if (elect_one_sync()) {
      constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t ID_O = idesc_bf16(128, D, false, true);
      const uint32_t sQ = sbase + L::Q_OFF;
      auto wait = [&](int b, uint32_t parity) {
        return mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag);
      };
      auto issue_s = [&](int jt) {
        const uint32_t sK = sbase + L::K_OFF + (jt & 1) * L::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + L::T_S + (jt % L::SBUF) * 128, fdesc_kmajor<D>(sQ, kk), fdesc_kmajor<D>(sK, kk),
                 ID_S, kk > 0);
        mma_commit(&bars[F_SFULL + jt % L::SBUF]);
        mma_commit(&bars[F_KEMPTY + (jt & 1)]);
      };
      bool ok = true;
      if (j_first < p.Tk && (ok = wait(F_Q, 0) && wait(F_KFULL, 0))) {
        tc_fence_after();
        issue_s(0);
        if (next_tile(j_first) < p.Tk && (ok = wait(F_KFULL + 1, 0))) issue_s(1);
      }
      for (int jt = 0, j = j_first; ok && j < p.Tk; ++jt, j = next_tile(j)) {
        const uint32_t sV = sbase + L::V_OFF + (jt & 1) * L::TILE;
        const uint32_t pbuf = tmem + L::T_S + (jt % L::SBUF) * 128;
        // O_g += P_j[:, group g's 64 keys] V_j[those keys], each half as soon
        // as its group has written it
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          if (!(ok = wait(F_PFULL + 2 * g + (jt & 1), (jt >> 1) & 1))) break;
          if (g == 0 && !(ok = wait(F_VFULL + (jt & 1), (jt >> 1) & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * g; kk < 4 * g + 4; ++kk)
            mma_ts(tmem + L::T_O + g * D, pbuf + fp_col(16 * kk), fdesc_mnmajor<D>(sV, kk),
                   ID_O, (jt > 0 || kk > 4 * g));
          mma_commit(&bars[(g == 0 ? F_PVDONE : F_PVDONE1) + (jt & 1)]);
        }
        if (!ok) break;
        mma_commit(&bars[F_VEMPTY + (jt & 1)]);
        if (next_tile(next_tile(j)) < p.Tk) {
          // S_{j+2} overwrites P_{j+2-SBUF}, which that tile's P V reads
          const int jo = jt + 2 - L::SBUF;
          if (jo >= 0 && !(ok = wait(F_PVDONE1 + (jo & 1), (jo >> 1) & 1))) break;
          if (!(ok = wait(F_KFULL + (jt & 1), ((jt + 2) >> 1) & 1))) break;
          tc_fence_after();
          issue_s(jt + 2);
        }
      }
      if (!ok) fail();
      mma_commit(&bars[F_FINAL]);
      mbar_wait(&bars[F_FINAL], 0, p.wait_cycles, never);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------ softmax warpgroups
    const int t = threadIdx.x & 127;
    const int g = threadIdx.x >> 7;
    const int qrow = i0 + t;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // Wait outcomes are made warp-uniform: the TMEM accesses are warp-collective.
    auto wait_w = [&](int b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(&bars[b], parity, p.wait_cycles, abort_flag));
    };
    float m = -INFINITY, z = 0.f;
    bool ok = true;
    int jt = 0;
    for (int j = j_first; j < p.Tk; ++jt, j = next_tile(j)) {
      const int kb = j * kTile + 64 * g;  // first key of this thread's 64 columns
      // keys with local index >= lim are excluded for this row: keys past
      // N_k, keys after the query's position (causal), and in a kind-2 tile
      // of a block mask keys after the query inside the tile
      int lim = p.Nk - kb;
      if constexpr (kMask) {
        if (tile_kind(j) == 2 && t - 64 * g + 1 < lim) lim = t - 64 * g + 1;
      } else {
        if (p.causal && p.q_off + qrow - kb + 1 < lim) lim = p.q_off + qrow - kb + 1;
      }
      const bool masked = __any_sync(0xffffffffu, lim < 64);
      if (!(ok = wait_w(F_SFULL + jt % L::SBUF, (jt / L::SBUF) & 1))) break;
      tc_fence_after();
      const uint32_t sbuf = lane_base + L::T_S + (jt % L::SBUF) * 128;
      uint32_t sr[64];
      tmem_ld32(sbuf + 64 * g, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(sbuf + 64 * g + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_ld_wait(sr);
      float mx = -INFINITY;
      if (masked) {
#pragma unroll
        for (int u = 0; u < 64; ++u)
          if (u < lim) mx = fmaxf(mx, __uint_as_float(sr[u]));
      } else {
#pragma unroll
        for (int u = 0; u < 64; ++u) mx = fmaxf(mx, __uint_as_float(sr[u]));
      }
      mx *= p.scale_log2;  // the tile's maximum over this half-row, log2 units
      float alpha = 1.f;
      const bool raise = mx > m + kRescaleMargin;
      if (raise) {
        alpha = jt > 0 ? ex2_approx(m - mx) : 1.f;
        m = mx;
      }
      if (__any_sync(0xffffffffu, raise && jt > 0)) {
        // O_g holds this group's sum_{j' < j} P_j' V_j' with the old m: scale
        // it by alpha once the last of those products has landed.
        const int done = g == 1 ? F_PVDONE1 : F_PVDONE;
        if (!(ok = wait_w(done + ((jt - 1) & 1), ((jt - 1) >> 1) & 1))) break;
        tc_fence_after();
        const uint32_t o_cols = L::T_O + g * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 16) {
          uint32_t ov[16];
          tmem_ld16(lane_base + o_cols + c, ov);
          tmem_ld_wait(ov);
#pragma unroll
          for (int u = 0; u < 16; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
          tmem_st16(lane_base + o_cols + c, ov);
        }
        z *= alpha;
      }
      // P = exp2(S * scale*log2e - m) -> bf16 into the first 32 of this group's
      // columns. The arguments are formed two at a time by a packed FMA; one
      // pair in four is exponentiated on the FMA pipe (exp2_fma2), the rest
      // on MUFU, whose 16 results per clock per SM would otherwise take twice
      // as long as the tile's two MMAs at d = 64.
      uint32_t pk[32];
      float zt = 0.f;
      const uint64_t c2 = f2(p.scale_log2, p.scale_log2), nm2 = f2(-m, -m);
#pragma unroll
      for (int u = 0; u < 64; u += 2) {
        const float2 x =
            f2_split(fma2(f2(__uint_as_float(sr[u]), __uint_as_float(sr[u + 1])), c2, nm2));
        float p0, p1;
        if ((u / 2) % 4 == 3) {
          const float2 e = exp2_fma2(x.x, x.y);
          p0 = e.x;
          p1 = e.y;
        } else {
          p0 = ex2_approx(x.x);
          p1 = ex2_approx(x.y);
        }
        if (masked) {
          if (u >= lim) p0 = 0.f;
          if (u + 1 >= lim) p1 = 0.f;
        }
        zt += p0 + p1;
        pk[u / 2] = pack_bf16x2(p0, p1);
      }
      z += zt;
      tmem_st16(sbuf + fp_col(64 * g), *reinterpret_cast<uint32_t(*)[16]>(pk));
      tmem_st16(sbuf + fp_col(64 * g) + 16, *reinterpret_cast<uint32_t(*)[16]>(pk + 16));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars[F_PFULL + 2 * g + (jt & 1)]);
    }
    // Epilogue: the last P V has landed; combine the two halves' sums. A
    // query tile that meets no key tile has O = 0 and LSE = -inf (the log of
    // an empty sum).
    const int n_kv = jt;
    if (ok && n_kv > 0) ok = wait_w(F_PVDONE1 + ((n_kv - 1) & 1), ((n_kv - 1) >> 1) & 1);
    // weights of this group's O_g (a_own) and of the other's (a_oth)
    float a_own = 1.f, a_oth = 0.f;
    if (ok && n_kv > 0) {
      xm[g * 128 + t] = m;
      xm[256 + g * 128 + t] = z;
      mbar_arrive(&bars[F_XCHG]);
      ok = wait_w(F_XCHG, 0);
      if (ok) {
        const float m2 = xm[(g ^ 1) * 128 + t], z2 = xm[256 + (g ^ 1) * 128 + t];
        const float mm = fmaxf(m, m2);
        // a group none of whose keys the row sees has m = -inf, z = 0
        a_own = m == -INFINITY ? 0.f : ex2_approx(m - mm);
        a_oth = m2 == -INFINITY ? 0.f : ex2_approx(m2 - mm);
        z = z * a_own + z2 * a_oth;
        m = mm;
      }
    }
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      const float inv = z > 0.f ? 1.f / z : 0.f;
      const bool row_ok = qrow < p.N && CSA_IN_BOUNDS(bh < p.BH && it_q < p.T, p.status);
      __nv_bfloat16* orow =
          p.o + p.os.row(bh, row_ok ? qrow : 0) + g * L::HALF_D;
#pragma unroll 1
      for (int c = 0; c < L::HALF_D; c += 16) {
        uint32_t ov[16];
        if (n_kv > 0) {
          // channels [g*d/2 + c, +16) of a_0 O_0 + a_1 O_1
          uint32_t o0[16], o1[16];
          tmem_ld16(lane_base + L::T_O + g * L::HALF_D + c, o0);
          tmem_ld16(lane_base + L::T_O + D + g * L::HALF_D + c, o1);
          tmem_ld_wait(o0, o1);
          const float a0 = g == 0 ? a_own : a_oth, a1 = g == 0 ? a_oth : a_own;
#pragma unroll
          for (int u = 0; u < 16; ++u)
            ov[u] = __float_as_uint(__uint_as_float(o0[u]) * a0 + __uint_as_float(o1[u]) * a1);
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) ov[u] = 0u;
        }
        if (row_ok) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[8 * v]) * inv, __uint_as_float(ov[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ov[8 * v + 2]) * inv, __uint_as_float(ov[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ov[8 * v + 4]) * inv, __uint_as_float(ov[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ov[8 * v + 6]) * inv, __uint_as_float(ov[8 * v + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c + 8 * v) = w;
          }
        }
      }
      if (row_ok && g == 0)
        p.lse[static_cast<size_t>(bh) * p.N + qrow] =
            z > 0.f ? (m + __log2f(z)) * 0.6931471805599453f : -INFINITY;
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
cudaError_t launch_fwd_d(const TmaMaps& m, void* o, float* lse, int* status, int BH,
                         const Extent& ex, bool causal, float scale, const uint8_t* bmask,
                         const RowStrides& os, cudaStream_t s) {
  using L = FwdLayout<D>;
  static_assert(L::ALLOC <= 232448, "shared memory window exceeds 227 KB");
  auto kern = bmask ? attn_fwd_bf16_sm100_kernel<D, true> : attn_fwd_bf16_sm100_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = status;
  p.N = ex.nq;
  p.T = (ex.nq + kTile - 1) / kTile;
  p.BH = BH;
  p.Nk = ex.nk;
  p.Tk = (ex.nk + kTile - 1) / kTile;
  p.q_off = ex.q_off;
  // Heads per group: as many as fit, with their K and V tiles, in about a
  // third of L2.
  int dev = 0, l2 = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0)
    l2 = 126 << 20;
  const size_t head_bytes = static_cast<size_t>(p.Tk) * kTile * D * 4;
  p.G = static_cast<int>(std::max<size_t>(1, std::min<size_t>(BH, (l2 / 3) / head_bytes)));
  p.causal = causal ? 1 : 0;
  p.bmask = bmask;
  p.os = os;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_cycles = kWaitLimitCycles;
  const unsigned grid = static_cast<unsigned>(p.T) * static_cast<unsigned>(BH);
  kern<<<grid, kFwdThreads, L::ALLOC, s>>>(m.a, m.b, m.c, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const TmaMaps& maps, void* o, float* lse, int* status, int BH,
                            const Extent& ex, int d, bool causal, float scale,
                            const uint8_t* block_mask, const RowStrides& os, cudaStream_t s) {
  switch (d) {
    case 32: return launch_fwd_d<32>(maps, o, lse, status, BH, ex, causal, scale, block_mask, os, s);
    case 64: return launch_fwd_d<64>(maps, o, lse, status, BH, ex, causal, scale, block_mask, os, s);
    case 128:
      return launch_fwd_d<128>(maps, o, lse, status, BH, ex, causal, scale, block_mask, os, s);
    default: return cudaErrorInvalidValue;
  }
}

namespace {
// Test hook: the forward's two exponentials side by side, 2^x by
// exp2_fma2 (FMA pipe) and by ex2.approx (MUFU), for n inputs.
__global__ void exp2_pair_kernel(const float* __restrict__ x, float* __restrict__ poly,
                                 float* __restrict__ mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  const float2 e = sm100::exp2_fma2(a, b);
  poly[i] = e.x;
  mufu[i] = sm100::ex2_approx(a);
  if (i + 1 < n) {
    poly[i + 1] = e.y;
    mufu[i + 1] = sm100::ex2_approx(b);
  }
}
}  // namespace

cudaError_t launch_exp2_pair(const float* x, float* poly, float* mufu, int n, cudaStream_t s) {
  const int pairs = (n + 1) / 2;
  exp2_pair_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(x, poly, mufu, n);
  return cudaGetLastError();
}

}  // namespace csa
