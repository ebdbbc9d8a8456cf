// Forward of causal softmax attention on the sm_100a tensor cores (tcgen05).
//
// One CTA per (query tile i of 128 rows, head bh). For each key tile j that
// the causal filter lets tile i see (j <= i):
//
//   S   = Q_i K_j^T                    (tcgen05 MMA -> TMEM, lane = query row)
//   m   = max(m, rowmax S * scale*log2e);  P = exp2(S * scale*log2e - m)
//   z   = z * exp2(m_old - m) + rowsum P   (one thread per row, CUDA cores)
//   O_j = P V_j                        (tcgen05 MMA -> TMEM), O = O*alpha + O_j
//
// and writes O = O / z (bf16) and LSE = (m + log2 z) * ln 2, the one saved
// number per row of ddx issue #243 (item 2). The max-shifted softmax is the
// `weights` / `norm` steps of ddx issue #217's repro; the key filter is its
// `WHERE q.pos >= k.pos` (diagonal kept).
//
// Warp roles as in the backward: warps 0-3 own one query row each (TMEM lane
// = row), warp 4 issues TMA loads and MMAs from one elected lane.
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {

__device__ int g_fwd_status;  // forward's status word (per device)

int* fwd_status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fwd_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

namespace {

using namespace sm100;

template <int D>
struct FwdLayout {
  static constexpr int CH = D >= 64 ? 64 : D;
  static constexpr int NCH = D / CH;
  static constexpr int ROWB = CH * 2;
  static constexpr int CHUNK = kTile * ROWB;
  static constexpr int TILE = NCH * CHUNK;
  static constexpr uint32_t SWZ = ROWB == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr int STAGES = 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;                 // [STAGES] tiles
  static constexpr int V_OFF = K_OFF + STAGES * TILE;        // [STAGES] tiles
  static constexpr int P_OFF = V_OFF + STAGES * TILE;        // [128 q][128 k] bf16
  static constexpr int BAR_OFF = P_OFF + 32768;
  static constexpr int MISC_OFF = BAR_OFF + 16 * 8;
  static constexpr int BYTES = MISC_OFF + 64;
  static constexpr int ALLOC = (BYTES + 1024) > 118 * 1024 ? (BYTES + 1024) : 118 * 1024;
  static constexpr uint32_t T_S = 0, T_O = 128;
  static constexpr uint32_t T_COLS = 256;
};

enum FBar { F_Q = 0, F_KVFULL = 1, F_KVEMPTY = 3, F_SFULL = 5, F_PFULL, F_OFULL, F_OREAD,
            F_FINAL, F_COUNT };

struct FwdParams {
  __nv_bfloat16* o;  // [BH][N][D]
  float* lse;        // [BH][N]
  int* status;
  int N, T, BH;
  int causal;
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
__device__ __forceinline__ uint64_t fdesc_p_kmajor(uint32_t tile, int kk) {
  const int e = kk * 16;
  return smem_desc(tile + (e / 64) * 16384 + (e % 64) * 2, 16, 1024, kSwizzle128B);
}
__device__ __forceinline__ uint32_t fp_offset(int r, int g) {
  return (g >> 3) * 16384 + r * 128 + (((g & 7) ^ (r & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(160, 1)
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

  const int warp = threadIdx.x >> 5;
  // longest-first: the last query tiles see the most key tiles
  const int it_q = p.causal ? (p.T - 1 - static_cast<int>(blockIdx.x) / p.BH)
                            : static_cast<int>(blockIdx.x) / p.BH;
  const int bh = blockIdx.x % p.BH;
  const int i0 = it_q * kTile;
  const int n_kv = p.causal ? it_q + 1 : p.T;

  if (threadIdx.x == 0) {
    mbar_init(&bars[F_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[F_KVFULL + s], 1);
      mbar_init(&bars[F_KVEMPTY + s], 1);
    }
    mbar_init(&bars[F_SFULL], 1);
    mbar_init(&bars[F_PFULL], 128);
    mbar_init(&bars[F_OFULL], 1);
    mbar_init(&bars[F_OREAD], 128);
    mbar_init(&bars[F_FINAL], 1);
    *abort_flag = 0;
    *const_cast<volatile int*>(never) = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_base_slot, L::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(p.status, kStatusTimeout);
  };

  if (warp == 4) {
    if (elect_one_sync()) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(&bars[F_Q], L::TILE);
      for (int c = 0; c < L::NCH; ++c)
        tma_load_3d(smem + L::Q_OFF + c * L::CHUNK, &tm_q, &bars[F_Q], c * L::CH, i0, bh);
      auto load_kv = [&](int jt) {
        const int s = jt & 1;
        uint64_t* bar = &bars[F_KVFULL + s];
        mbar_arrive_expect_tx(bar, 2 * L::TILE);
        for (int c = 0; c < L::NCH; ++c) {
          tma_load_3d(smem + L::K_OFF + s * L::TILE + c * L::CHUNK, &tm_k, bar, c * L::CH,
                      jt * kTile, bh);
          tma_load_3d(smem + L::V_OFF + s * L::TILE + c * L::CHUNK, &tm_v, bar, c * L::CH,
                      jt * kTile, bh);
        }
      };
      int loaded = 0, waited = 0;
      for (int jt = 0; jt < n_kv && jt < 2; ++jt, ++loaded) load_kv(jt);
      constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t ID_O = idesc_bf16(128, D, false, true);
      const uint32_t sQ = sbase + L::Q_OFF, sP = sbase + L::P_OFF;
      bool ok = mbar_wait(&bars[F_Q], 0, p.wait_cycles, abort_flag);
      const bool q_waited = ok;
      for (int jt = 0; ok && jt < n_kv; ++jt) {
        const int s = jt & 1;
        const uint32_t ph = (jt >> 1) & 1;
        const uint32_t sK = sbase + L::K_OFF + s * L::TILE;
        const uint32_t sV = sbase + L::V_OFF + s * L::TILE;
        if (!(ok = mbar_wait(&bars[F_KVFULL + s], ph, p.wait_cycles, abort_flag))) break;
        ++waited;
        // S may be overwritten once the row threads have read S(jt-1) (they
        // arrive on F_PFULL after that).
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + L::T_S, fdesc_kmajor<D>(sQ, kk), fdesc_kmajor<D>(sK, kk), ID_S, kk > 0);
        mma_commit(&bars[F_SFULL]);
        if (!(ok = mbar_wait(&bars[F_PFULL], jt & 1, p.wait_cycles, abort_flag))) break;
        // O_j lands where the threads read O_(jt-1); they arrive on F_OREAD after.
        if (jt > 0 && !(ok = mbar_wait(&bars[F_OREAD], (jt - 1) & 1, p.wait_cycles, abort_flag)))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + L::T_O, fdesc_p_kmajor(sP, kk), fdesc_mnmajor<D>(sV, kk), ID_O, kk > 0);
        mma_commit(&bars[F_OFULL]);
        mma_commit(&bars[F_KVEMPTY + s]);
        if (jt + 2 < n_kv) {
          if (!(ok = mbar_wait(&bars[F_KVEMPTY + s], ph, p.wait_cycles, abort_flag))) break;
          load_kv(jt + 2);
          ++loaded;
        }
      }
      if (!ok) {
        fail();
        if (!q_waited) mbar_wait(&bars[F_Q], 0, p.wait_cycles, never);
        for (int w = waited; w < loaded; ++w)
          mbar_wait(&bars[F_KVFULL + (w & 1)], (w >> 1) & 1, p.wait_cycles, never);
      }
      mma_commit(&bars[F_FINAL]);
      mbar_wait(&bars[F_FINAL], 0, p.wait_cycles, never);
    }
    __syncwarp();
  } else {
    const int t = threadIdx.x;
    const int qrow = i0 + t;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float o[D];
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] = 0.f;
    float m = -INFINITY, z = 0.f;
    // Wait outcomes are made warp-uniform: the TMEM loads are warp-collective.
    auto wait_w = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.wait_cycles, abort_flag));
    };
    bool ok = true;
    uint8_t* sP = smem + L::P_OFF;
    for (int jt = 0; jt < n_kv; ++jt) {
      const int j0 = jt * kTile;
      // keys with local index >= lim are excluded for this row
      int lim = p.N - j0;
      if (p.causal && qrow - j0 + 1 < lim) lim = qrow - j0 + 1;
      if (!(ok = wait_w(&bars[F_SFULL], jt & 1))) break;
      tc_fence_after();
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_base + L::T_S + 32 * c, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int u = 0; u < 32; ++u)
          if (32 * c + u < lim) mx = fmaxf(mx, __uint_as_float(r[u]));
      }
      const float m_new = fmaxf(m, mx * p.scale_log2);
      // rows that have seen no key yet keep m = -inf; guard the -inf - -inf case
      const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m - m_new);
      const float msub = (m_new == -INFINITY) ? 0.f : m_new;
      float zt = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_base + L::T_S + 32 * c, r);
        tmem_ld_wait(r);
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 32; u += 2) {
          float p0 = ex2_approx(fmaf(__uint_as_float(r[u]), p.scale_log2, -msub));
          float p1 = ex2_approx(fmaf(__uint_as_float(r[u + 1]), p.scale_log2, -msub));
          if (32 * c + u >= lim) p0 = 0.f;
          if (32 * c + u + 1 >= lim) p1 = 0.f;
          zt += p0 + p1;
          pk[u / 2] = pack_bf16x2(p0, p1);
        }
#pragma unroll
        for (int v = 0; v < 4; ++v)
          st_shared_v4(smem_u32(sP) + fp_offset(t, 4 * c + v), pk[4 * v], pk[4 * v + 1],
                       pk[4 * v + 2], pk[4 * v + 3]);
      }
      z = z * alpha + zt;
      m = m_new;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[F_PFULL]);
      if (!(ok = wait_w(&bars[F_OFULL], jt & 1))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_base + L::T_O + 32 * c, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int u = 0; u < 32; ++u) o[32 * c + u] = fmaf(o[32 * c + u], alpha, __uint_as_float(r[u]));
      }
      tc_fence_before();
      mbar_arrive(&bars[F_OREAD]);
    }
    if (!ok) {
      fail();
    } else if (qrow < p.N) {
      const float inv = 1.f / z;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + qrow) * D;
#pragma unroll
      for (int c = 0; c < D; c += 8) {
        uint4 v;
        v.x = pack_bf16x2(o[c] * inv, o[c + 1] * inv);
        v.y = pack_bf16x2(o[c + 2] * inv, o[c + 3] * inv);
        v.z = pack_bf16x2(o[c + 4] * inv, o[c + 5] * inv);
        v.w = pack_bf16x2(o[c + 6] * inv, o[c + 7] * inv);
        *reinterpret_cast<uint4*>(orow + c) = v;
      }
      p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m + __log2f(z)) * 0.6931471805599453f;
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
cudaError_t launch_fwd_d(const TmaMaps& m, void* o, float* lse, int* status, int BH, int N,
                         bool causal, float scale, cudaStream_t s) {
  using L = FwdLayout<D>;
  auto kern = attn_fwd_bf16_sm100_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = status;
  p.N = N;
  p.T = (N + kTile - 1) / kTile;
  p.BH = BH;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_cycles = kWaitLimitCycles;
  const unsigned grid = static_cast<unsigned>(p.T) * static_cast<unsigned>(BH);
  kern<<<grid, 160, L::ALLOC, s>>>(m.a, m.b, m.c, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const TmaMaps& maps, void* o, float* lse, int* status, int BH, int N,
                            int d, bool causal, float scale, cudaStream_t s) {
  switch (d) {
    case 32: return launch_fwd_d<32>(maps, o, lse, status, BH, N, causal, scale, s);
    case 64: return launch_fwd_d<64>(maps, o, lse, status, BH, N, causal, scale, s);
    case 128: return launch_fwd_d<128>(maps, o, lse, status, BH, N, causal, scale, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa
