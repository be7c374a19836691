// fa_fwd_sm100.cu -- bf16 attention forward on B200 tensor cores (tcgen05).
//
// What it computes ("FlashAttention-2: Faster Attention with Better
// Parallelism and Work Partitioning" review page, core-algorithm answer,
// section 2 (1) tiling and (2) forward pass; "IO-4 FlashAttention" note,
// sections 3-4): for every query tile Q_i (128 rows) it visits the key/value
// tiles K_j, V_j (128 rows each), forms S_ij = Q_i K_j^T on the tensor
// cores, keeps a running row max m and running row sum l, accumulates the
// unnormalised output, and divides by l once at the end (the deferred
// rescaling the review lists as FA2's reduction of non-matmul work).  S and
// P never leave the SM: S lives in tensor memory (TMEM), P is written back
// over S as bf16 and fed to the second MMA straight from TMEM.
//
// B200 design (one CTA per 128-row query tile, 6 warps):
//   warp 4      TMA producer: Q tile once, then K_j and V_j into separate
//               3- or 4-stage shared-memory rings (mbarrier full/empty pairs).
//   warp 5      TMEM allocator and single-thread MMA issuer:
//               S_j = Q K_j^T into TMEM buffer j%2 (SS form), then
//               O += P_{j-1} V_{j-1} with P read from TMEM (TS form), so the
//               tensor core computes S_j while the softmax works on S_{j-1}.
//   warps 0-3   softmax: one thread per query row (= TMEM lane).  Base-2
//               domain, lazy rescaling: the reference max is only moved
//               (and O, l rescaled in TMEM) when the row max grew by more
//               than 2^8, which keeps every exponent <= 8 and makes O
//               corrections rare after the first tiles.  They also run the
//               epilogue (O / l -> bf16, LSE).
// Causal: tiles above the diagonal are never loaded; only the diagonal tile
// and a ragged last tile are masked.  CTAs run group-major (a few heads at a
// time, so their K and V stay in L2), longest-first inside a group.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace fwd {

constexpr int kBM = 128;              // query rows per tile (TMEM lanes)
constexpr int kBN = 128;              // keys per K/V tile
constexpr int kThreads = 192;         // 4 softmax warps + producer + MMA
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (log2 units)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;       // O accumulator columns [256, 256+d)

template <int D>
struct Cfg {
  static constexpr int NB = (D + 63) / 64;  // 64-column (128-byte) swizzle blocks
  static constexpr int BLK = 64 * kBM * 2;  // bytes of one 128 x 64 bf16 block
  static constexpr int TILE = NB * BLK;     // bytes of one Q/K/V tile
  static constexpr int NST = NB == 1 ? 4 : 3;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + NST * TILE;
  static constexpr int BAR_OFF = V_OFF + NST * TILE;
  static constexpr int NBAR = 1 + 4 * NST + 2 + 2 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;  // + slack for 1 KB alignment
  static constexpr int KSTEPS = D / 16;
  static_assert(D % 16 == 0 && D <= 128, "head dim must be a multiple of 16, <= 128");
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Drain wait used only while aborting: ignores the abort flag, bounded by time.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(a, parity)) {
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      atomicCAS(ctl.status, 0, kSiteFwdDrain);
      return;
    }
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
               float* __restrict__ lse, int N, int BH, int group, float scale_log2,
               WaitCtl ctl) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::NST;
  uint64_t* v_full = k_empty + C::NST;
  uint64_t* v_empty = v_full + C::NST;
  uint64_t* s_full = v_empty + C::NST;  // [2]
  uint64_t* p_full = s_full + 2;        // [2]
  uint64_t* o_done = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = warp_id();
  const int lane = lane_id();
  const int n_kv_all = (N + kBN - 1) / kBN;
  // Group-major order: `group` heads at a time (their K and V stay in L2),
  // and inside a group the longest query tiles first, head fastest.
  int bh, qt;
  {
    const int per_group = group * n_kv_all;
    const int g = static_cast<int>(blockIdx.x) / per_group;
    const int r = static_cast<int>(blockIdx.x) - g * per_group;
    const int gh = min(group, BH - g * group);
    const int t = r / gh;
    qt = n_kv_all - 1 - t;
    bh = g * group + (r - t * gh);
  }
  const int n_kv = CAUSAL ? min(qt + 1, n_kv_all) : n_kv_all;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, kBM);
    }
    mbar_init(o_done, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int last_k[C::NST], last_v[C::NST];
#pragma unroll
      for (int s = 0; s < C::NST; ++s) last_k[s] = last_v[s] = -1;
      mbar_arrive_expect_tx(q_full, C::TILE);
#pragma unroll
      for (int b = 0; b < C::NB; ++b)
        tma_load_3d(&tm_q, q_full, smem + C::Q_OFF + b * C::BLK, b * 64, qt * kBM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % C::NST;
        const uint32_t u = static_cast<uint32_t>(j / C::NST);
        if (j >= C::NST && !mbar_wait(k_empty + s, (u - 1) & 1, abort, ctl, kSiteFwdProducer))
          break;
        mbar_arrive_expect_tx(k_full + s, C::TILE);
#pragma unroll
        for (int b = 0; b < C::NB; ++b)
          tma_load_3d(&tm_k, k_full + s, smem + C::K_OFF + s * C::TILE + b * C::BLK, b * 64,
                      j * kBN, bh);
        last_k[s] = static_cast<int>(u);
        if (j >= C::NST && !mbar_wait(v_empty + s, (u - 1) & 1, abort, ctl, kSiteFwdProducer))
          break;
        mbar_arrive_expect_tx(v_full + s, C::TILE);
#pragma unroll
        for (int b = 0; b < C::NB; ++b)
          tma_load_3d(&tm_v, v_full + s, smem + C::V_OFF + s * C::TILE + b * C::BLK, b * 64,
                      j * kBN, bh);
        last_v[s] = static_cast<int>(u);
      }
      if (*abort) {
        // Let every copy this CTA started land before shared memory is released.
        drain_wait(q_full, 0, ctl);
        for (int s = 0; s < C::NST; ++s) {
          if (last_k[s] >= 0) drain_wait(k_full + s, last_k[s] & 1, ctl);
          if (last_v[s] >= 0) drain_wait(v_full + s, last_v[s] & 1, ctl);
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16(kBM, D, 0, 1);
      const uint32_t q_addr = sbase + C::Q_OFF;
      auto issue_pv = [&](int t) -> bool {
        const int sb = t & 1;
        if (!mbar_wait(p_full + sb, (t >> 1) & 1, abort, ctl, kSiteFwdMma)) return false;
        const int s = t % C::NST;
        if (!mbar_wait(v_full + s, (t / C::NST) & 1, abort, ctl, kSiteFwdMma)) return false;
        tc_fence_after();
        const uint32_t v_addr = sbase + C::V_OFF + s * C::TILE;
        const uint32_t p_tmem = tmem + sb * kBN;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // V_j as the K x N (keys x d) operand, d contiguous: MN-major.
          const uint64_t bdesc = sdesc_sw128(v_addr + kk * 16 * 128, C::BLK, 1024);
          mma_ts(tmem + kColO, p_tmem + kk * 8, bdesc, kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(v_empty + s);
        mma_commit(o_done);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, abort, ctl, kSiteFwdMma);
      tc_fence_after();
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % C::NST;
        if (!mbar_wait(k_full + s, (j / C::NST) & 1, abort, ctl, kSiteFwdMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = sbase + C::K_OFF + s * C::TILE;
        const uint32_t s_tmem = tmem + (j & 1) * kBN;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(s_tmem, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                 kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full + (j & 1));
        mma_commit(k_empty + s);
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(n_kv - 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax (warps 0..3)
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int q_idx = qt * kBM + r;
    float m = -INFINITY;  // reference max, base-2 scaled units
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      const bool w = mbar_wait(s_full + sb, (j >> 1) & 1, abort, ctl, kSiteFwdSoftmax);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
      {
        uint32_t t0[32], t1[32];
        tmem_ld32(lane_base + sb * kBN + 0, t0);
        tmem_ld32(lane_base + sb * kBN + 32, t1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = __uint_as_float(t0[c]);
          s[32 + c] = __uint_as_float(t1[c]);
        }
        tmem_ld32(lane_base + sb * kBN + 64, t0);
        tmem_ld32(lane_base + sb * kBN + 96, t1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[64 + c] = __uint_as_float(t0[c]);
          s[96 + c] = __uint_as_float(t1[c]);
        }
      }
      const int kv0 = j * kBN;
      const bool diag = CAUSAL && (j == n_kv - 1);
      if (diag || kv0 + kBN > N) {
        const int lim = min(N - kv0, CAUSAL ? (q_idx - kv0 + 1) : kBN);  // visible keys
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < kBN; ++c) mx = fmaxf(mx, s[c]);
      const float m_cand = fmaxf(m, mx * scale_log2);
      const bool grow = m_cand > m + kRescaleLog2;  // true on the first tile
      const float alpha = grow ? ex2(m - m_cand) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O must hold P_{j-1} V_{j-1} before it is rescaled.
        const bool w2 = mbar_wait(o_done, (j - 1) & 1, abort, ctl, kSiteFwdSoftmax);
        if (!__all_sync(0xffffffffu, w2)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t o16[16];
          tmem_ld16(lane_base + kColO + c * 16, o16);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o16[e] = __float_as_uint(__uint_as_float(o16[e]) * alpha);
          tmem_st16(lane_base + kColO + c * 16, o16);
        }
        tmem_wait_st();
      }
      if (grow) {
        l *= alpha;
        m = m_cand;
      }
      const float neg_m = (m == -INFINITY) ? 0.f : -m;
      float rs = 0.f;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN / 2; ++c) {
        const float p0 = ex2(fmaf(s[2 * c], scale_log2, neg_m));
        const float p1 = ex2(fmaf(s[2 * c + 1], scale_log2, neg_m));
        rs += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l += rs;
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
        tmem_st32(lane_base + sb * kBN + 0, lo);
        tmem_st32(lane_base + sb * kBN + 32, hi);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full + sb);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) {
      const bool w = mbar_wait(o_done, (n_kv - 1) & 1, abort, ctl, kSiteFwdEpilogue);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        const float inv_l = 1.f / l;
        const bool valid = q_idx < N;
        uint4* orow = reinterpret_cast<uint4*>(out + (static_cast<size_t>(bh) * N + q_idx) * D);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t o16[16];
          tmem_ld16(lane_base + kColO + c * 16, o16);
          tmem_wait_ld();
          uint4 a, b;
          a.x = pack_bf16(__uint_as_float(o16[0]) * inv_l, __uint_as_float(o16[1]) * inv_l);
          a.y = pack_bf16(__uint_as_float(o16[2]) * inv_l, __uint_as_float(o16[3]) * inv_l);
          a.z = pack_bf16(__uint_as_float(o16[4]) * inv_l, __uint_as_float(o16[5]) * inv_l);
          a.w = pack_bf16(__uint_as_float(o16[6]) * inv_l, __uint_as_float(o16[7]) * inv_l);
          b.x = pack_bf16(__uint_as_float(o16[8]) * inv_l, __uint_as_float(o16[9]) * inv_l);
          b.y = pack_bf16(__uint_as_float(o16[10]) * inv_l, __uint_as_float(o16[11]) * inv_l);
          b.z = pack_bf16(__uint_as_float(o16[12]) * inv_l, __uint_as_float(o16[13]) * inv_l);
          b.w = pack_bf16(__uint_as_float(o16[14]) * inv_l, __uint_as_float(o16[15]) * inv_l);
          if (valid) {
            orow[2 * c] = a;
            orow[2 * c + 1] = b;
          }
        }
        if (valid) lse[static_cast<size_t>(bh) * N + q_idx] = (m + __log2f(l)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool CAUSAL>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                   float* lse, int BH, int N, float scale, const Launch& L) {
  using C = Cfg<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(fwd_kernel<D, CAUSAL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_qt = (N + kBM - 1) / kBM;
  // Heads per group: keep a group's Q, K, V and O (8 N d bytes per head)
  // within ~48 MB of the 126 MB L2.
  const long long per_head = 8LL * N * D;
  int group = static_cast<int>((48LL << 20) / (per_head > 0 ? per_head : 1));
  group = group < 1 ? 1 : (group > BH ? BH : group);
  const long long blocks = static_cast<long long>(BH) * n_qt;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const float scale_log2 = scale * 1.4426950408889634f;
  WaitCtl ctl{L.status, L.limit_ns};
  fwd_kernel<D, CAUSAL><<<static_cast<unsigned>(blocks), kThreads, C::SMEM, L.stream>>>(
      tq, tk, tv, static_cast<__nv_bfloat16*>(o), lse, N, BH, group, scale_log2, ctl);
  return cudaGetLastError();
}

}  // namespace fwd

cudaError_t launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             void* o, float* lse, int BH, int N, int d, float scale, int causal,
                             const Launch& L) {
  switch (d) {
    case 64:
      return causal ? fwd::launch<64, true>(tq, tk, tv, o, lse, BH, N, scale, L)
                    : fwd::launch<64, false>(tq, tk, tv, o, lse, BH, N, scale, L);
    case 80:
      return causal ? fwd::launch<80, true>(tq, tk, tv, o, lse, BH, N, scale, L)
                    : fwd::launch<80, false>(tq, tk, tv, o, lse, BH, N, scale, L);
    case 128:
      return causal ? fwd::launch<128, true>(tq, tk, tv, o, lse, BH, N, scale, L)
                    : fwd::launch<128, false>(tq, tk, tv, o, lse, BH, N, scale, L);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace fa
