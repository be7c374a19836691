// fa_fwd64_sm100.cu -- bf16 attention forward with 64-key tiles and a
// double-buffered score tile (tcgen05).
//
// Same computation as fa_fwd_sm100.cu ("FlashAttention-2: Faster Attention
// with Better Parallelism and Work Partitioning" review page, core-algorithm
// answer, sections 2 (1) tiling and (2) forward pass): per 128-row query tile
// a running row max m and row sum l, the unnormalised output accumulated in
// tensor memory, one division by l at the end.  What differs is the block
// size of the key dimension, one of the parameters the review's
// implementation-cost answer, section (2), and its auto-tuning answer,
// section 1 (1), leave to be chosen per GPU: key tiles of 64 instead of 128.
//
// Why 64 on B200: with d = 128 the 512 TMEM columns hold exactly two 128 x 128
// fp32 score tiles and two 128 x 128 output accumulators, so with 128-key
// tiles S_x(j+1) can only be written after O_x += P_x(j) V_j has read P_x(j)
// (P lives over S): every key step of a query tile runs the chain softmax ->
// P V and S MMAs -> softmax, and the two tiles of a CTA together cannot hide
// it.  A 64-key score tile takes 64 columns, so each query tile gets two
// score buffers: S_x(j+2) is computed while the softmax works on S_x(j+1),
// the softmax of a tile runs step after step, and the tensor core works on
// whatever tile has operands ready.
//
// Work item: a pair of 128-row query tiles (A = 2p, B = 2p+1) of one head, as
// in the 128-key kernel; persistent CTAs take items through cluster launch
// control, group-major and longest-first.  12 warps:
//   warp 8      TMA producer: Q_A, Q_B once per item, then 64-key K and V
//               tiles into separate rings (each serves both query tiles).
//   warp 9      TMEM allocator and MMA issuer: per key step j and tile x,
//               O_x (+)= P_x(j) V_j, then S_x(j+2) = Q_x K_{j+2}^T into the
//               buffer P_x(j) occupied (issued after the P V that reads it).
//   warps 0-3 / 4-7  softmax of tile A / B: one thread per query row, base-2
//               domain, lazy rescaling (threshold 2^8), epilogue through
//               per-warp staging and TMA stores.
//   warps 10-11 idle (their registers go to the softmax warpgroups).
// TMEM: S_A buffers [0,64) and [64,128), S_B [128,192) and [192,256),
// O_A [256,256+d), O_B [384,384+d); P (bf16) is written over its S buffer.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace fwd64 {

constexpr int kBM = 128;       // query rows per tile (TMEM lanes)
constexpr int kBN = 64;        // keys per K/V tile
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;  // 216 + 216 + 72 = 3 x 168
constexpr int kControlRegs = 3 * kLaunchRegs - 2 * kSoftmaxRegs;
static_assert(2 * kSoftmaxRegs + kControlRegs <= 3 * kLaunchRegs, "register split over budget");
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int NB = (D + 63) / 64;      // 64-column (128-byte) swizzle blocks
  static constexpr int QBLK = kBM * 128;        // 128 rows x 64 bf16
  static constexpr int QTILE = NB * QBLK;
  static constexpr int KBLK = kBN * 128;        // 64 rows x 64 bf16
  static constexpr int KTILE = NB * KBLK;
  static constexpr int NST = NB == 1 ? 8 : 4;   // K and V ring stages
  static constexpr int Q_OFF = 0;               // [2] tiles A, B
  static constexpr int K_OFF = Q_OFF + 2 * QTILE;
  static constexpr int V_OFF = K_OFF + NST * KTILE;
  static constexpr int STG_OFF = V_OFF + NST * KTILE;  // [8 softmax warps] 4 KB O staging
  static constexpr int STG = 4096;
  static constexpr int BAR_OFF = STG_OFF + 8 * STG;
  // q_full, q_empty, k/v full/empty rings, s_full[2][2], p_full[2][2],
  // o_done[2][2], next-item full/empty [2] each
  static constexpr int NBAR = 2 + 4 * NST + 4 + 4 + 4 + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM = MISC_OFF + 48 + 1024;
  static constexpr int KSTEPS = D / 16;
  static_assert(D % 16 == 0 && D <= 128, "head dim must be a multiple of 16, <= 128");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(MISC_OFF % 16 == 0, "next-item responses need 16-byte alignment");
};

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

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         const WaitCtl& ctl, int site) {
  const bool w = mbar_wait(bar, parity, abort, ctl, site);
  return __all_sync(0xffffffffu, w);
}

// (bh, tile pair) of work item idx (group-major, longest pairs first, head
// fastest) and the 64-key tiles each query tile of the pair visits (0 for a
// tile past N): causal, keys below min(128 (qt + 1), N); otherwise all N.
template <bool CAUSAL>
__device__ __forceinline__ void decode_item(int idx, int N, int BH, int group, int& bh, int& pair,
                                            int (&n_x)[2]) {
  const int n_t = (N + kBM - 1) / kBM;
  const int n_pair = (n_t + 1) / 2;
  const int per_group = group * n_pair;
  const int g = idx / per_group;
  const int r = idx - g * per_group;
  const int gh = min(group, BH - g * group);
  const int t = r / gh;
  pair = n_pair - 1 - t;
  bh = g * group + (r - t * gh);
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int qt = 2 * pair + x;
    const int keys = CAUSAL ? min(kBM * (qt + 1), N) : N;
    n_x[x] = qt >= n_t ? 0 : (keys + kBN - 1) / kBN;
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd64_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 float* __restrict__ lse, int N, int BH, int group, float scale_log2,
                 WaitCtl ctl) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;          // the item's last S MMAs are done with Q_A, Q_B
  uint64_t* k_full = bars + 2;           // [NST]
  uint64_t* k_empty = k_full + C::NST;   // [NST]
  uint64_t* v_full = k_empty + C::NST;   // [NST]
  uint64_t* v_empty = v_full + C::NST;   // [NST]
  uint64_t* s_full = v_empty + C::NST;   // [tile x][buffer b] at s_full + 2 x + b
  uint64_t* p_full = s_full + 4;         // [x][b]: the four softmax warps wrote P
  uint64_t* o_done = p_full + 4;         // [x][parity of the P V's index]
  uint64_t* nxt_full = o_done + 4;       // [2] next-item requests
  uint64_t* nxt_empty = nxt_full + 2;    // [2]
  uint8_t* nxt_resp = smem + C::MISC_OFF;  // [2] x 16 bytes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF + 32);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 36);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, 4);  // one arrival per softmax warp of the tile
      mbar_init(o_done + b, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(nxt_full + b, 1);
      mbar_init(nxt_empty + b, 9);  // MMA warp + 8 softmax warps
    }
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto next_item = [&](int i, int& idx, int site) -> bool {
    return next_work_item(i, idx, nxt_full, nxt_empty, nxt_resp, abort, ctl, site);
  };

  if (warp >= 8) {
    regs_decrease<kControlRegs>();
    if (warp == 8) {
      // ------------------------------------------------------------ producer
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int last_k[C::NST], last_v[C::NST];
#pragma unroll
      for (int s = 0; s < C::NST; ++s) last_k[s] = last_v[s] = -1;
      int q_issued = 0;
      int nxt_pending = -1;
      uint32_t nxt_pending_par = 0;
      uint32_t kv = 0;  // K/V ring uses so far
      int idx = static_cast<int>(blockIdx.x);
      bool ok = true;
      for (int i = 0; ok; ++i) {
        if (i > 0) {
          if (!producer_take_item(i, idx, nxt_full, nxt_resp, abort, ctl, kSiteFwdProducer)) break;
          nxt_pending = -1;
          if (idx < 0) break;
        }
        // Ask for item i + 1 right away, so its loads follow this item's.
        if (!producer_request_item(i, nxt_full, nxt_empty, nxt_resp, abort, ctl, kSiteFwdProducer,
                                   leader, nxt_pending, nxt_pending_par))
          break;
        int bh, pair, n_x[2];
        decode_item<CAUSAL>(idx, N, BH, group, bh, pair, n_x);
        const int n_max = max(n_x[0], n_x[1]);
        if (n_max == 0) continue;
        if (q_issued > 0 &&
            !wait_all(q_empty, static_cast<uint32_t>(q_issued - 1) & 1, abort, ctl,
                      kSiteFwdProducer))
          break;
        if (leader) {
          const int nq = n_x[1] > 0 ? 2 : 1;
          mbar_arrive_expect_tx(q_full, nq * C::QTILE);
          for (int x = 0; x < nq; ++x)
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
              tma_load_3d(&tm_q, q_full, smem + C::Q_OFF + x * C::QTILE + b * C::QBLK, b * 64,
                          (2 * pair + x) * kBM, bh);
        }
        __syncwarp();
        ++q_issued;
        for (int j = 0; j < n_max; ++j, ++kv) {
          const int s = static_cast<int>(kv % C::NST);
          const uint32_t u = kv / C::NST;
          if (kv >= C::NST && !wait_all(k_empty + s, (u - 1) & 1, abort, ctl, kSiteFwdProducer)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(k_full + s, C::KTILE);
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
              tma_load_3d(&tm_k, k_full + s, smem + C::K_OFF + s * C::KTILE + b * C::KBLK,
                          b * 64, j * kBN, bh);
          }
          __syncwarp();
          last_k[s] = static_cast<int>(u);
          if (kv >= C::NST && !wait_all(v_empty + s, (u - 1) & 1, abort, ctl, kSiteFwdProducer)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(v_full + s, C::KTILE);
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
              tma_load_3d(&tm_v, v_full + s, smem + C::V_OFF + s * C::KTILE + b * C::KBLK,
                          b * 64, j * kBN, bh);
          }
          __syncwarp();
          last_v[s] = static_cast<int>(u);
        }
      }
      if (*abort && leader) {
        if (q_issued > 0) drain_wait(q_full, static_cast<uint32_t>(q_issued - 1) & 1, ctl);
        for (int s = 0; s < C::NST; ++s) {
          if (last_k[s] >= 0) drain_wait(k_full + s, last_k[s] & 1, ctl);
          if (last_v[s] >= 0) drain_wait(v_full + s, last_v[s] & 1, ctl);
        }
        if (nxt_pending >= 0) drain_wait(nxt_full + nxt_pending, nxt_pending_par, ctl);
      }
      __syncwarp();
    } else if (warp == 9) {
      // ---------------------------------------------------------- MMA issuer
      const bool leader = elect_one();
      constexpr uint32_t kIdescS = idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16(kBM, D, 0, 1);
      const SDesc q_desc = sdesc(sbase + C::Q_OFF, 16, 1024);      // K-major
      const SDesc k_desc = sdesc(sbase + C::K_OFF, 16, 1024);      // K-major
      const SDesc v_desc = sdesc(sbase + C::V_OFF, C::KBLK, 1024); // MN-major
      uint32_t kv_base = 0;   // K/V ring uses before this item
      uint32_t gs[2] = {0u, 0u};  // key steps of each tile before this item
      int k_seen = -1;
      auto wait_k = [&](int r) -> bool {  // ring use r has landed
        if (r <= k_seen) return true;
        if (!wait_all(k_full + r % C::NST, static_cast<uint32_t>(r / C::NST) & 1, abort, ctl,
                      kSiteFwdMma))
          return false;
        k_seen = r;
        tc_fence_after();
        return true;
      };
      // S_x = Q_x K^T (K in ring use r) into buffer b of tile x
      auto issue_s = [&](int x, int r, uint32_t b) {
        if (leader) {
          const SDesc qd = q_desc + x * C::QTILE;
          const SDesc kd = k_desc + (r % C::NST) * C::KTILE;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            mma_ss(tmem + x * 128 + b * kBN, qd + ((kk >> 2) * C::QBLK + (kk & 3) * 32),
                   kd + ((kk >> 2) * C::KBLK + (kk & 3) * 32), kIdescS, kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full + 2 * x + b);
        }
        __syncwarp();
      };
      // O_x (+)= P_x V (V in ring use r, P in buffer b); the commit goes to
      // the o_done barrier of this P V's index parity
      auto issue_pv = [&](int x, int r, uint32_t b, uint32_t opar, bool first) {
        if (leader) {
          const SDesc vd = v_desc + (r % C::NST) * C::KTILE;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts(tmem + 256 + x * 128, tmem + x * 128 + b * kBN + kk * 8, vd + kk * 16 * 128,
                   kIdescPV, (!first || kk > 0) ? 1u : 0u);
          mma_commit(o_done + 2 * x + opar);
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (leader) mma_commit(bar);
        __syncwarp();
      };
      bool ok = true;
      int idx = 0;
      uint32_t q_items = 0;
      for (int i = 0; ok; ++i) {
        if (!next_item(i, idx, kSiteFwdMma)) break;
        if (idx < 0) break;
        int bh, pair, n_x[2];
        decode_item<CAUSAL>(idx, N, BH, group, bh, pair, n_x);
        const int n_max = max(n_x[0], n_x[1]);
        if (n_max == 0) continue;
        const int r0 = static_cast<int>(kv_base);
        ok = wait_all(q_full, q_items & 1, abort, ctl, kSiteFwdMma);
        ++q_items;
        if (!ok) break;
        tc_fence_after();
        // Prologue: the first two score tiles of each query tile.
        for (int jj = 0; ok && jj < 2 && jj < n_max; ++jj) {
          if (!wait_k(r0 + jj)) {
            ok = false;
            break;
          }
          for (int x = 0; x < 2; ++x)
            if (jj < n_x[x]) issue_s(x, r0 + jj, (gs[x] + jj) & 1);
          commit(k_empty + (r0 + jj) % C::NST);
        }
        if (!ok) break;
        if (n_max <= 2) commit(q_empty);
        for (int j = 0; ok && j < n_max; ++j) {
          const int r = r0 + j;
          if (!wait_all(v_full + r % C::NST, static_cast<uint32_t>(r / C::NST) & 1, abort, ctl,
                        kSiteFwdMma)) {
            ok = false;
            break;
          }
          for (int x = 0; ok && x < 2; ++x) {
            if (j >= n_x[x]) continue;
            const uint32_t g = gs[x] + j;
            if (!wait_all(p_full + 2 * x + (g & 1), (g >> 1) & 1, abort, ctl, kSiteFwdMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(x, r, g & 1, g & 1, j == 0);
            if (j + 2 < n_x[x]) {
              if (!wait_k(r + 2)) {
                ok = false;
                break;
              }
              issue_s(x, r + 2, g & 1);  // after the P V that read this buffer
            }
          }
          if (!ok) break;
          commit(v_empty + r % C::NST);
          if (j + 2 < n_max) commit(k_empty + (r + 2) % C::NST);
          if (j + 3 == n_max) commit(q_empty);  // the item's last S MMAs are issued
        }
        kv_base += static_cast<uint32_t>(n_max);
        gs[0] += static_cast<uint32_t>(n_x[0]);
        gs[1] += static_cast<uint32_t>(n_x[1]);
      }
      __syncwarp();
    }
  } else {
    regs_increase<kSoftmaxRegs>();
    // --------------------------------------- softmax (warps 0-3: A, 4-7: B)
    const int x = warp >> 2;
    const int r = threadIdx.x & 127;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t col_o = 256 + x * 128;
    uint32_t gs = 0;  // key steps of this tile before the current item
    bool ok = true;
    int idx = 0;
    for (int i = 0; ok; ++i) {
      if (!next_item(i, idx, kSiteFwdSoftmax)) break;
      if (idx < 0) break;
      int bh, pair, n_x[2];
      decode_item<CAUSAL>(idx, N, BH, group, bh, pair, n_x);
      const int n_kv = n_x[x];
      if (n_kv == 0) continue;  // this tile lies past N
      const int qt_x = 2 * pair + x;
      const int q_idx = qt_x * kBM + r;
      float m = -INFINITY;  // reference max, base-2 scaled units
      float l = 0.f;
      for (int j = 0; j < n_kv; ++j) {
        const uint32_t g = gs + j;
        const uint32_t b = g & 1;
        const uint32_t col_s = x * 128 + b * kBN;
        if (!wait_all(s_full + 2 * x + b, (g >> 1) & 1, abort, ctl, kSiteFwdSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[kBN];
        {
          uint32_t t0[32], t1[32];
          tmem_ld32(lane_base + col_s, t0);
          tmem_ld32(lane_base + col_s + 32, t1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            s[c] = __uint_as_float(t0[c]);
            s[32 + c] = __uint_as_float(t1[c]);
          }
        }
        const int kv0 = j * kBN;
        const bool masked = (CAUSAL && kv0 + kBN - 1 > qt_x * kBM) || kv0 + kBN > N;
        const int lim = masked ? min(N - kv0, CAUSAL ? (q_idx - kv0 + 1) : kBN) : kBN;
        if (masked) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        const float mx = row_max(s);
        const float m_cand = fmaxf(m, mx * scale_log2);
        const bool grow = m_cand > m + kRescaleLog2;  // true on the first tile
        // Rare after an item's first steps: some row of this warp moves its
        // reference max (no exponential on the common path).
        if (__any_sync(0xffffffffu, grow)) {
          const float alpha = grow ? ex2(m - m_cand) : 1.f;
          if (j > 0) {
            // O_x must hold every earlier P V before it is rescaled: wait for
            // the P V of step j - 1 (the one before it completed before S_x(j)).
            const uint32_t pv = g - 1;
            if (!wait_all(o_done + 2 * x + (pv & 1), (pv >> 1) & 1, abort, ctl, kSiteFwdSoftmax)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
              uint32_t o16[16];
              tmem_ld16(lane_base + col_o + c * 16, o16);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e)
                o16[e] = __float_as_uint(__uint_as_float(o16[e]) * alpha);
              tmem_st16(lane_base + col_o + c * 16, o16);
            }
          }
          if (grow) {
            l *= alpha;
            m = m_cand;
          }
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const float2 sc2 = make_float2(scale_log2, scale_log2);
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        uint32_t pk[kBN / 2];
#pragma unroll
        for (int c = 0; c < kBN / 2; ++c) {
          const float2 xx = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
          const float2 p = make_float2(ex2(xx.x), ex2(xx.y));
          rs2[c & 3] = __fadd2_rn(rs2[c & 3], p);
          pk[c] = pack_bf16(p.x, p.y);
        }
        const float2 rsa = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
        l += rsa.x + rsa.y;
        tmem_st32(lane_base + col_s, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + 2 * x + b);
      }
      // -------------------------------------------------------- epilogue
      const uint32_t pv_last = gs + n_kv - 1;
      if (ok && wait_all(o_done + 2 * x + (pv_last & 1), (pv_last >> 1) & 1, abort, ctl,
                         kSiteFwdEpilogue)) {
        tc_fence_after();
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const float lse_row = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        // This warp's 32 rows of O, 64 columns per TMA store (columns past d
        // and rows past N are not written), staged in its own 4 KB swizzled
        // buffer: row `lane`, 16-byte chunk c at chunk c ^ (lane % 8).
        const int row0 = qt_x * kBM + (warp & 3) * 32;
#pragma unroll
        for (int b = 0; b < C::NB; ++b) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          const uint32_t rowa = sbase + C::STG_OFF + warp * C::STG + lane * 128;
#pragma unroll
          for (int hf = 0; hf < 4; ++hf) {
            uint32_t t[16];
            tmem_ld16(lane_base + col_o + 64 * b + 16 * hf, t);
            tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 2; ++c4) {
              const int c = 2 * hf + c4, e0 = 8 * c4;
              st_shared_v4(rowa + ((c ^ (lane & 7)) << 4),
                           pack_bf16(__uint_as_float(t[e0 + 0]) * inv_l,
                                     __uint_as_float(t[e0 + 1]) * inv_l),
                           pack_bf16(__uint_as_float(t[e0 + 2]) * inv_l,
                                     __uint_as_float(t[e0 + 3]) * inv_l),
                           pack_bf16(__uint_as_float(t[e0 + 4]) * inv_l,
                                     __uint_as_float(t[e0 + 5]) * inv_l),
                           pack_bf16(__uint_as_float(t[e0 + 6]) * inv_l,
                                     __uint_as_float(t[e0 + 7]) * inv_l));
            }
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0 && row0 < N) {
            tma_store_3d(&tm_o, smem + C::STG_OFF + warp * C::STG, 64 * b, row0, bh);
            bulk_commit();
          }
        }
        if (q_idx < N) lse[static_cast<size_t>(bh) * N + q_idx] = lse_row;
        // The next item's first P V (accumulate off) overwrites O_x only after
        // this warpgroup's next P, so the loads above are complete by then.
        tc_fence_before();
      } else if (ok) {
        ok = false;
      }
      gs += static_cast<uint32_t>(n_kv);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool CAUSAL>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& to, float* lse, int BH, int N, float scale,
                   const Launch& L) {
  using C = Cfg<D>;
  static bool configured = false;
  if (!configured) {
    // The register split assumes exactly kLaunchRegs per thread at launch.
    cudaFuncAttributes fattr;
    cudaError_t e = cudaFuncGetAttributes(&fattr, fwd64_kernel<D, CAUSAL>);
    if (e != cudaSuccess) return e;
    if (fattr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(fwd64_kernel<D, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_t = (N + kBM - 1) / kBM;
  const int n_pair = (n_t + 1) / 2;
  // Heads per group as in the 128-key kernel: K and V of a head (4 N d
  // bytes) are what its items re-read.
  const long long per_head = 4LL * N * D;
  int group = static_cast<int>(l2_group_bytes(CAUSAL) / (per_head > 0 ? per_head : 1));
  group = group < 1 ? 1 : (group > BH ? BH : group);
  const long long blocks = static_cast<long long>(BH) * n_pair;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  WaitCtl ctl{L.status, L.limit_ns};
  fwd64_kernel<D, CAUSAL><<<static_cast<unsigned>(blocks), kThreads, C::SMEM, L.stream>>>(
      tq, tk, tv, to, lse, N, BH, group, scale * 1.4426950408889634f, ctl);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& to, float* lse, int BH, int N, float scale, int causal,
                     const Launch& L) {
  return causal ? launch<D, true>(tq, tk, tv, to, lse, BH, N, scale, L)
                : launch<D, false>(tq, tk, tv, to, lse, BH, N, scale, L);
}

}  // namespace fwd64

cudaError_t launch_fwd64_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& to, float* lse, int BH, int N, int d,
                               float scale, int causal, const Launch& L) {
  switch (d) {
    case 64:
      return fwd64::launch_d<64>(tq, tk, tv, to, lse, BH, N, scale, causal, L);
    case 80:
      return fwd64::launch_d<80>(tq, tk, tv, to, lse, BH, N, scale, causal, L);
    case 128:
      return fwd64::launch_d<128>(tq, tk, tv, to, lse, BH, N, scale, causal, L);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace fa
