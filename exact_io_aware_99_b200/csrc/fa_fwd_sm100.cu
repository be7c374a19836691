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
// B200 design: a work item is a pair of 128-row query tiles (A = 2p,
// B = 2p+1) of one head; the grid has one CTA per item, and a running CTA
// takes further items by cancelling CTAs that have not started yet (cluster
// launch control), so one CTA per SM works through items in launch order and
// the rings, barriers and TMEM carry over from one item to the next.
// 12 warps (warps 10-11 idle; the third warpgroup gives its registers to the
// two softmax warpgroups):
//   warp 8      TMA producer: both Q tiles of an item, then K_j and V_j into
//               separate shared-memory rings; each K/V tile serves both Q
//               tiles (half the K/V traffic per FLOP of a one-tile CTA).  It
//               requests the next item as soon as it starts the current one,
//               so the next item's loads follow the current item's without a
//               gap.
//   warp 9      TMEM allocator and MMA issuer (one elected lane), alternating
//               between the tiles: O_A += P_A V_j, S_A = Q_A K_{j+1}^T,
//               O_B += P_B V_j, S_B = Q_B K_{j+1}^T, so the tensor core works
//               on one tile while the other tile's softmax runs.
//   warps 0-3   softmax of tile A, warps 4-7 softmax of tile B: one thread
//               per query row (= TMEM lane), base-2 domain, lazy rescaling
//               (the reference max moves, and O and l are rescaled in TMEM,
//               only when the row max grew by more than 2^8; exponents stay
//               <= 8).  P leaves in two halves (keys 0-63, then 64-127),
//               each with its own barrier, so the P V MMA starts on the first
//               half while the second half is exponentiated (measured +1-2 %;
//               four quarters cost more in barriers than they gain).  They
//               also run their tile's epilogue (O / l, LSE):
//               each warp writes its 32 rows of O, 64 columns at a time,
//               into its own 4 KB swizzled staging buffer and one lane
//               stores it with TMA (whole rows per transfer instead of one
//               16-byte piece of 32 different rows per store instruction).
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+d),
// O_B [384,384+d).  S of a tile is single-buffered: S_X(j+1) is issued after
// O_X += P_X(j) V_j, so when the softmax sees S_X(j+1) the previous P V has
// completed and O_X can be rescaled without waiting.
// Causal: tiles above the diagonal are never loaded; only the diagonal tile
// and a ragged last tile are masked.  CTAs run group-major (a few heads at a
// time, so their K and V stay in L2), longest-first inside a group.
#include <cuda_bf16.h>

#include <type_traits>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace fwd {

constexpr int kBM = 128;              // query rows per tile (TMEM lanes)
constexpr int kBN = 128;              // keys per K/V tile
constexpr int kThreads = 384;         // 2 softmax warpgroups + producer/MMA warpgroup
// Registers per thread: 168 at launch (384 threads), then the softmax
// warpgroups take RegSplit::kSoftmax each and the producer/MMA warpgroup keeps the
// rest: 224 + 224 + 56 = 504 = 3 x 168, the launch budget of each lane slot.
// With a block mask the producer walks the mask with its whole warp and
// needs more, so the split is 216 + 216 + 72.
constexpr int kLaunchRegs = 168;
template <bool BS>
struct RegSplit {
  static constexpr int kSoftmax = BS ? 216 : 224;
  static constexpr int kControl = 3 * kLaunchRegs - 2 * kSoftmax;
  static_assert(2 * kSoftmax + kControl <= 3 * kLaunchRegs, "register split over budget");
};
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (log2 units)
// One column pair in FA_FWD_POLY_EVERY uses the FMA-pipe exp2 (0: none).
// Measured on B200 with P in two halves: 1 in 8 +1.1 % (N = 4096 causal),
// +1.9 % (N = 16384), +2.2 % (d = 80); 1 in 16 +1.1 / +1.3 %; 1 in 4 slower.
#ifndef FA_FWD_POLY_EVERY
#define FA_FWD_POLY_EVERY 8
#endif
constexpr int kPolyMod = FA_FWD_POLY_EVERY > 0 ? FA_FWD_POLY_EVERY : 1;
#ifndef FA_FWD_P_PARTS
#define FA_FWD_P_PARTS 2
#endif
// P of a step leaves the softmax in kPParts equal parts (kPCols bf16 pairs,
// i.e. 2 kPCols keys, each with its own barrier), so the P V MMA starts on
// the first keys while the last exponentials are still being computed.
constexpr int kPParts = FA_FWD_P_PARTS;
constexpr int kPCols = kBN / 2 / kPParts;
static_assert(kPParts >= 1 && kPCols % 16 == 0 && kPCols * kPParts == kBN / 2, "P parts");
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int NB = (D + 63) / 64;  // 64-column (128-byte) swizzle blocks
  static constexpr int BLK = 64 * kBM * 2;  // bytes of one 128 x 64 bf16 block
  static constexpr int TILE = NB * BLK;     // bytes of one Q/K/V tile
  static constexpr int NST = NB == 1 ? 4 : 2;
  static constexpr int Q_OFF = 0;           // [2] tiles A, B
  static constexpr int K_OFF = Q_OFF + 2 * TILE;
  static constexpr int V_OFF = K_OFF + NST * TILE;
  static constexpr int STG_OFF = V_OFF + NST * TILE;  // [8 softmax warps] 4 KB O staging
  static constexpr int STG = 4096;                     // 32 rows x 64 bf16 columns
  static constexpr int BAR_OFF = STG_OFF + 8 * STG;
  static constexpr int NBAR = 2 + 4 * NST + 4 + 2 * kPParts + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // 16-byte aligned (next-item responses)
  static constexpr int SMEM = MISC_OFF + 48 + 1024;    // + slack for 1 KB alignment
  static constexpr int KSTEPS = D / 16;
  static_assert(D % 16 == 0 && D <= 128, "head dim must be a multiple of 16, <= 128");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(MISC_OFF % 16 == 0, "next-item responses need 16-byte alignment");
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

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         const WaitCtl& ctl, int site) {
  const bool w = mbar_wait(bar, parity, abort, ctl, site);
  return __all_sync(0xffffffffu, w);
}

// (bh, tile pair) and the key tiles each of the pair's query tiles visits
// (0 when tile B lies past N), for work item `idx` in group-major order:
// `group` heads at a time (their K and V stay in L2), and inside a group the
// longest tile pairs first, head fastest.
template <bool CAUSAL>
__device__ __forceinline__ void decode_item(int idx, int n_t, int BH, int group, int& bh,
                                            int& pair, int (&n_x)[2]) {
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
    n_x[x] = qt >= n_t ? 0 : (CAUSAL ? min(qt + 1, n_t) : n_t);
  }
}

// Key tiles of one work item when a block mask is given (block-sparse
// attention): tile x of the pair (query tile qt[x]) sees key tile j when the
// tile exists, j <= qt[x] if causal, and the mask byte (qt[x], j) is set.
// The pair visits the union of its two tiles' key tiles; a tile that does not
// see a visited key tile treats that step as fully masked.
template <bool CAUSAL>
struct ItemTiles {
  const uint8_t* row[2];  // mask rows of the two query tiles
  int qt[2];
  bool has[2];
  int n_t;
  __device__ __forceinline__ bool active(int x, int j) const {
    return has[x] && (!CAUSAL || j <= qt[x]) && row[x][j] != 0;
  }
  __device__ __forceinline__ bool any(int j) const { return active(0, j) || active(1, j); }
  // Bit b of word w: key tile 32 w + b is visited.  Called by all 32 lanes
  // of a converged warp (each lane reads one tile's mask bytes).
  __device__ __forceinline__ uint32_t word(int w) const {
    const int j = 32 * w + lane_id();
    return __ballot_sync(0xffffffffu, j < n_t && any(j));
  }
};


// Steps of a work item and, with a block mask, the tiles it visits.  Dense:
// tile x visits key tiles [0, n_x[x]); block-sparse: both tiles step through
// the union of visited key tiles (n_x[1] = 0 when tile B lies past N).
template <bool CAUSAL, bool BS>
__device__ __forceinline__ void item_plan(int idx, int n_t, int BH, int group, int H,
                                          const uint8_t* bmask, int mask_heads, int& bh,
                                          int& pair, int (&n_x)[2], ItemTiles<CAUSAL>& it) {
  decode_item<CAUSAL>(idx, n_t, BH, group, bh, pair, n_x);
  if (BS) {
    const int hm = mask_heads == 1 ? 0 : bh % H;
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      it.qt[x] = 2 * pair + x;
      it.has[x] = it.qt[x] < n_t;
      it.row[x] = bmask + (static_cast<size_t>(hm) * n_t + (it.has[x] ? it.qt[x] : 0)) * n_t;
    }
    it.n_t = n_t;
    int steps = 0;
    for (int w = 0; w < (n_t + 31) / 32; ++w) steps += __popc(it.word(w));
    n_x[0] = steps;
    n_x[1] = it.has[1] ? steps : 0;
  }
}

__device__ __forceinline__ int floor_div(int a, int b) {
  return a >= 0 ? a / b : -((-a + b - 1) / b);
}

// Split-KV items (decode): item idx = (tile pair item, split) with the split
// fastest.  The split covers key tiles [t0, t0 + kt_per) of the N_k keys;
// tile x visits the ones it sees (causal: keys <= query + coff, coff =
// N_k - N_q, so the last query sees every key).
template <bool CAUSAL>
__device__ __forceinline__ void split_plan(int idx, int n_t, int BH, int group,
                                           const SplitKv& sk, int& bh, int& pair, int& t0,
                                           int (&n_x)[2]) {
  decode_item<CAUSAL>(idx / sk.n_split, n_t, BH, group, bh, pair, n_x);
  const int n_kt = (sk.Nk + kBN - 1) / kBN;
  t0 = (idx % sk.n_split) * sk.kt_per;
  const int t1 = min(t0 + sk.kt_per, n_kt);
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int qt = 2 * pair + x;
    int end = t1;
    if (CAUSAL) end = min(t1, floor_div(qt * kBM + kBM - 1 + sk.coff, kBN) + 1);
    n_x[x] = qt >= n_t ? 0 : max(0, end - t0);
  }
}

template <int D, bool CAUSAL, bool BS, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               __nv_bfloat16* __restrict__ out,
               float* __restrict__ lse, int N, int BH, int group, float scale_log2,
               const uint8_t* __restrict__ bmask, int mask_heads, int H, SplitKv sk,
               WaitCtl ctl) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;         // Q tiles no longer read by the item's S MMAs
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::NST;
  uint64_t* v_full = k_empty + C::NST;
  uint64_t* v_empty = v_full + C::NST;
  uint64_t* s_full = v_empty + C::NST;  // [2] per tile
  uint64_t* p_full = s_full + 2;        // [2 tiles][kPParts parts of P]
  uint64_t* o_done = p_full + 2 * kPParts;  // [2] per tile
  // Next-item requests (cluster launch control), double-buffered: the
  // producer issues the request for item i + 1 into slot (i + 1) & 1 once it
  // has issued item i's loads; the MMA warp and the 8 softmax warps read it
  // when they move on, and release the slot through nxt_empty.
  uint64_t* nxt_full = o_done + 2;      // [2]
  uint64_t* nxt_empty = nxt_full + 2;   // [2]
  uint8_t* nxt_resp = smem + C::MISC_OFF;  // [2] x 16 bytes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF + 32);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 36);

  const int warp = warp_id();
  const int lane = lane_id();
  // Query tiles (== key tiles, except for split-KV launches where the N_k
  // keys are counted by SplitKv).
  const int n_t = (N + kBN - 1) / kBN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full + x, 1);
      for (int q = 0; q < kPParts; ++q) mbar_init(p_full + kPParts * x + q, kBM);
      mbar_init(o_done + x, 1);
      mbar_init(nxt_full + x, 1);
      mbar_init(nxt_empty + x, 9);  // MMA warp + 8 softmax warps
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

  // Work item i of this CTA: its own index first, then the CTAs it
  // cancelled.  Consumers read the request the producer issued during item
  // i - 1 (use (i - 1) >> 1 of slot i & 1) and release the slot.  Returns
  // false when a wait gave up; idx < 0 means the grid has no work left.
  auto next_item = [&](int i, int& idx, int site) -> bool {
    if (i == 0) {
      idx = static_cast<int>(blockIdx.x);
      return true;
    }
    const int sl = i & 1;
    if (!wait_all(nxt_full + sl, static_cast<uint32_t>((i - 1) >> 1) & 1, abort, ctl, site))
      return false;
    idx = clc_result_x(nxt_resp + 16 * sl);
    __syncwarp();
    if (lane == 0) mbar_arrive(nxt_empty + sl);
    return true;
  };

  if (warp >= 8) {
  regs_decrease<RegSplit<BS>::kControl>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // Dense launches run the producer on one lane.  With a block mask the
    // whole warp runs the loop (it reads the mask with all lanes, see
    // ItemTiles::word) and the elected lane issues the copies and requests.
    auto produce = [&](auto warp_mode) {
      constexpr bool W = decltype(warp_mode)::value;
      const bool leader = W ? elect_one() : true;
      auto wait = [&](uint64_t* bar, uint32_t par) -> bool {
        return W ? wait_all(bar, par, abort, ctl, kSiteFwdProducer)
                 : mbar_wait(bar, par, abort, ctl, kSiteFwdProducer);
      };
      auto sync = [&]() {
        if (W) __syncwarp();
      };
      if (leader) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int last_k[C::NST], last_v[C::NST];
#pragma unroll
      for (int s = 0; s < C::NST; ++s) last_k[s] = last_v[s] = -1;
      int q_issued = 0;           // Q loads issued (one per item with work)
      int nxt_pending = -1;       // slot of a request in flight
      uint32_t nxt_pending_par = 0;
      uint32_t kv = 0;            // K/V ring uses so far
      int idx = static_cast<int>(blockIdx.x);
      bool ok = true;
      for (int i = 0; ok; ++i) {
        if (i > 0) {
          const int sl = i & 1;
          if (!wait(nxt_full + sl, static_cast<uint32_t>((i - 1) >> 1) & 1)) break;
          nxt_pending = -1;
          idx = clc_result_x(nxt_resp + 16 * sl);
          if (idx < 0) break;
        }
        // Ask for item i + 1 right away: its answer is then at hand when
        // this item's last loads are out, and the next Q can follow them.
        {
          const int sl1 = (i + 1) & 1;
          const uint32_t u1 = static_cast<uint32_t>(i >> 1);
          if (u1 > 0 && !wait(nxt_empty + sl1, (u1 - 1) & 1)) break;
          if (leader) {
            mbar_arrive_expect_tx(nxt_full + sl1, 16);
            clc_try_cancel(nxt_resp + 16 * sl1, nxt_full + sl1);
          }
          sync();
          nxt_pending = sl1;
          nxt_pending_par = u1 & 1;
        }
        int bh, pair, n_x[2];
        ItemTiles<CAUSAL> tiles;
        int t0 = 0;  // first key tile of a split-KV item
        if (SPLIT)
          split_plan<CAUSAL>(idx, n_t, BH, group, sk, bh, pair, t0, n_x);
        else
          item_plan<CAUSAL, BS>(idx, n_t, BH, group, H, bmask, mask_heads, bh, pair, n_x, tiles);
        const int n_max = max(n_x[0], n_x[1]);
        if (n_max > 0) {
          // Q of this item replaces the previous item's once its S MMAs are done.
          if (q_issued > 0 && !wait(q_empty, static_cast<uint32_t>(q_issued - 1) & 1)) break;
          if (leader) {
            const int nq = n_x[1] > 0 ? 2 : 1;
            mbar_arrive_expect_tx(q_full, nq * C::TILE);
            for (int x = 0; x < nq; ++x)
#pragma unroll
              for (int b = 0; b < C::NB; ++b)
                tma_load_3d(&tm_q, q_full, smem + C::Q_OFF + x * C::TILE + b * C::BLK, b * 64,
                            (2 * pair + x) * kBM, bh);
          }
          sync();
          ++q_issued;
          TileCursor cur(n_t);
          for (int j = 0; j < n_max; ++j, ++kv) {
            const int jt = BS ? cur.next(tiles) : t0 + j;  // key tile of the step
            const int s = static_cast<int>(kv % C::NST);
            const uint32_t u = kv / C::NST;
            if (kv >= C::NST && !wait(k_empty + s, (u - 1) & 1)) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_arrive_expect_tx(k_full + s, C::TILE);
#pragma unroll
              for (int b = 0; b < C::NB; ++b)
                tma_load_3d(&tm_k, k_full + s, smem + C::K_OFF + s * C::TILE + b * C::BLK,
                            b * 64, jt * kBN, bh);
            }
            sync();
            last_k[s] = static_cast<int>(u);
            if (kv >= C::NST && !wait(v_empty + s, (u - 1) & 1)) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_arrive_expect_tx(v_full + s, C::TILE);
#pragma unroll
              for (int b = 0; b < C::NB; ++b)
                tma_load_3d(&tm_v, v_full + s, smem + C::V_OFF + s * C::TILE + b * C::BLK,
                            b * 64, jt * kBN, bh);
            }
            sync();
            last_v[s] = static_cast<int>(u);
          }
          if (!ok) break;
        }
      }
      if (*abort && leader) {
        // Let every copy and request this CTA started land before shared
        // memory is released.
        if (q_issued > 0) drain_wait(q_full, static_cast<uint32_t>(q_issued - 1) & 1, ctl);
        for (int s = 0; s < C::NST; ++s) {
          if (last_k[s] >= 0) drain_wait(k_full + s, last_k[s] & 1, ctl);
          if (last_v[s] >= 0) drain_wait(v_full + s, last_v[s] & 1, ctl);
        }
        if (nxt_pending >= 0) drain_wait(nxt_full + nxt_pending, nxt_pending_par, ctl);
      }
    };
    if (BS)
      produce(std::true_type{});
    else if (lane == 0)
      produce(std::false_type{});
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    // The whole warp runs the schedule (waits and branches stay uniform);
    // the elected lane issues the MMAs and commits.
    const bool leader = elect_one();
    constexpr uint32_t kIdescS = idesc_bf16(kBM, kBN, 0, 0);
    constexpr uint32_t kIdescPV = idesc_bf16(kBM, D, 0, 1);
    const SDesc q_desc = sdesc(sbase + C::Q_OFF, 16, 1024);       // K-major
    const SDesc k_desc = sdesc(sbase + C::K_OFF, 16, 1024);       // K-major
    const SDesc v_desc = sdesc(sbase + C::V_OFF, C::BLK, 1024);   // MN-major
    uint32_t kv_base = 0;            // K/V ring uses before this item
    uint32_t p_base[2] = {0u, 0u};   // p_full phases consumed before this item
    int k_seen = -1;                 // highest ring use whose k_full wait was done
    auto wait_k = [&](int r) -> bool {  // ring use r
      if (r <= k_seen) return true;
      if (!wait_all(k_full + r % C::NST, static_cast<uint32_t>(r / C::NST) & 1, abort, ctl,
                    kSiteFwdMma))
        return false;
      k_seen = r;
      tc_fence_after();
      return true;
    };
    auto issue_s = [&](int x, int r) {  // S_x = Q_x K^T, K in ring use r
      if (leader) {
        const SDesc qd = q_desc + x * C::TILE;
        const SDesc kd = k_desc + (r % C::NST) * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + x * kBN, qd + off, kd + off, kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full + x);
      }
      __syncwarp();
    };
    // O_x (+)= P_x V over the keys of k-steps [K0, K1) (16 keys each), P_x
    // from TMEM; the last part signals o_done.
    auto issue_pv = [&](int x, int r, bool first, auto k0, auto k1) {
      constexpr int K0 = decltype(k0)::value, K1 = decltype(k1)::value;
      if (leader) {
        const SDesc vd = v_desc + (r % C::NST) * C::TILE;
#pragma unroll
        for (int kk = K0; kk < K1; ++kk)
          mma_ts(tmem + 256 + x * kBN, tmem + x * kBN + kk * 8, vd + kk * 16 * 128, kIdescPV,
                 (!first || kk > 0) ? 1u : 0u);
        if (K1 == kBN / 16) mma_commit(o_done + x);
      }
      __syncwarp();
    };
    auto commit = [&](uint64_t* bar) {
      if (leader) mma_commit(bar);
      __syncwarp();
    };
    bool ok = true;
    int idx = 0;
    uint32_t q_items = 0;  // items with at least one step (one Q load each)
    for (int i = 0; ok; ++i) {
      if (!next_item(i, idx, kSiteFwdMma)) break;
      if (idx < 0) break;
      int bh, pair, n_x[2];
      ItemTiles<CAUSAL> tiles;
      int t0 = 0;  // first key tile of a split-KV item
        if (SPLIT)
          split_plan<CAUSAL>(idx, n_t, BH, group, sk, bh, pair, t0, n_x);
        else
          item_plan<CAUSAL, BS>(idx, n_t, BH, group, H, bmask, mask_heads, bh, pair, n_x, tiles);
      const int n_max = max(n_x[0], n_x[1]);
      if (n_max == 0) continue;  // block mask hides the whole item
      const int r0 = static_cast<int>(kv_base);
      ok = wait_all(q_full, q_items & 1, abort, ctl, kSiteFwdMma) && wait_k(r0);
      ++q_items;
      if (!ok) break;
      tc_fence_after();
      for (int x = 0; x < 2; ++x)
        if (n_x[x] > 0) issue_s(x, r0);
      commit(k_empty + r0 % C::NST);
      if (n_max == 1) commit(q_empty);
      for (int j = 0; ok && j < n_max; ++j) {
        const int r = r0 + j;
        if (!wait_all(v_full + r % C::NST, static_cast<uint32_t>(r / C::NST) & 1, abort, ctl,
                      kSiteFwdMma)) {
          ok = false;
          break;
        }
        for (int x = 0; ok && x < 2; ++x) {
          if (j >= n_x[x]) continue;
          // P_x arrives in parts; each part's k-steps go as soon as it is in.
          bool got = true;
          static_for<kPParts>([&](auto q) {
            constexpr int Q = decltype(q)::value;
            if (!got) return;
            got = wait_all(p_full + kPParts * x + Q, (p_base[x] + j) & 1, abort, ctl,
                           kSiteFwdMma);
            if (!got) return;
            tc_fence_after();
            issue_pv(x, r, j == 0, std::integral_constant<int, Q * kPCols / 8>{},
                     std::integral_constant<int, (Q + 1) * kPCols / 8>{});
          });
          if (!got) {
            ok = false;
            break;
          }
          if (j + 1 < n_x[x]) {
            if (!wait_k(r + 1)) {
              ok = false;
              break;
            }
            issue_s(x, r + 1);
          }
        }
        if (!ok) break;
        commit(v_empty + r % C::NST);
        if (j + 1 < n_max) commit(k_empty + (r + 1) % C::NST);
        if (j + 2 == n_max) commit(q_empty);  // the item's last S MMAs are issued
      }
      kv_base += static_cast<uint32_t>(n_max);
      p_base[0] += static_cast<uint32_t>(n_x[0]);
      p_base[1] += static_cast<uint32_t>(n_x[1]);
    }
    __syncwarp();
  }
  } else {
    regs_increase<RegSplit<BS>::kSoftmax>();
    // --------------------------------------- softmax (warps 0-3: A, 4-7: B)
    const int x = warp >> 2;
    const int r = threadIdx.x & 127;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t col_s = x * kBN;
    const uint32_t col_o = 256 + x * kBN;

    uint32_t s_base = 0;  // s_full / o_done phases of this tile before the current item
    bool ok = true;
    int idx = 0;
    for (int i = 0; ok; ++i) {
      if (!next_item(i, idx, kSiteFwdSoftmax)) break;
      if (idx < 0) break;
      int bh, pair, n_x[2];
      ItemTiles<CAUSAL> tiles;
      int t0 = 0;  // first key tile of a split-KV item
        if (SPLIT)
          split_plan<CAUSAL>(idx, n_t, BH, group, sk, bh, pair, t0, n_x);
        else
          item_plan<CAUSAL, BS>(idx, n_t, BH, group, H, bmask, mask_heads, bh, pair, n_x, tiles);
      const int n_kv = n_x[x];
      const int qt_x = 2 * pair + x;
      const int q_idx = qt_x * kBM + r;
      // Split-KV launches write this split's partial (O normalised over the
      // split's keys, fp32, and its LSE) for the combine kernel.
      const size_t prow =
          SPLIT ? (static_cast<size_t>(idx % sk.n_split) * BH + bh) * N + q_idx : 0;
      if (n_kv == 0) {
        // No visible key for this tile (block mask, or a split past the
        // causal limit): O = 0, LSE = -inf.  (Dense launches only get here
        // for a tile past N: nothing to write.)
        if (q_idx < N) {
          if (SPLIT) {
            float4* prw = reinterpret_cast<float4*>(sk.part_o + prow * D);
#pragma unroll
            for (int c = 0; c < D / 4; ++c) prw[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            sk.part_lse[prow] = -INFINITY;
          } else {
            uint4* orow =
                reinterpret_cast<uint4*>(out + (static_cast<size_t>(bh) * N + q_idx) * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) orow[c] = make_uint4(0u, 0u, 0u, 0u);
            lse[static_cast<size_t>(bh) * N + q_idx] = -INFINITY;
          }
        }
        continue;
      }
      float m = -INFINITY;  // reference max, base-2 scaled units
      float l = 0.f;
      TileCursor cur(n_t);
      for (int j = 0; j < n_kv; ++j) {
        const int jt = BS ? cur.next(tiles) : t0 + j;  // key tile of the step
        if (!wait_all(s_full + x, (s_base + j) & 1, abort, ctl, kSiteFwdSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[kBN];
        {
          uint32_t t0[32], t1[32];
          tmem_ld32(lane_base + col_s + 0, t0);
          tmem_ld32(lane_base + col_s + 32, t1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            s[c] = __uint_as_float(t0[c]);
            s[32 + c] = __uint_as_float(t1[c]);
          }
          tmem_ld32(lane_base + col_s + 64, t0);
          tmem_ld32(lane_base + col_s + 96, t1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            s[64 + c] = __uint_as_float(t0[c]);
            s[96 + c] = __uint_as_float(t1[c]);
          }
        }
        const int kv0 = jt * kBN;
        bool masked;
        int lim;
        if (SPLIT) {
          // N_k keys, query q sees keys <= q + coff when causal
          masked = (CAUSAL && kv0 + kBN - 1 > qt_x * kBM + sk.coff) || kv0 + kBN > sk.Nk;
          lim = masked ? min(sk.Nk - kv0, CAUSAL ? (q_idx + sk.coff - kv0 + 1) : kBN) : kBN;
        } else {
          const bool act = !BS || tiles.active(x, jt);  // false: the mask hides the whole step
          const bool diag = CAUSAL && (BS ? jt == qt_x : j == n_kv - 1);
          masked = !act || diag || kv0 + kBN > N;
          lim = !act ? 0 : (masked ? min(N - kv0, CAUSAL ? (q_idx - kv0 + 1) : kBN) : kBN);
        }
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
            // O_x += P_x(j-1) V completed before S_x(j) (same MMA thread, in
            // order), so O_x can be rescaled now.
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
        // One column pair in FA_FWD_POLY_EVERY goes to the FMA-pipe exp2, the
        // rest to the special-function unit, so the two units share the work.
        float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        uint32_t pk[kBN / 2];
        auto exp_pair = [&](int c) {
          const float2 xx = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
          float2 p;
          if (FA_FWD_POLY_EVERY > 0 && c % kPolyMod == kPolyMod - 1) {
            p = exp2_fma2(xx);
            if (masked) {
              if (2 * c >= lim) p.x = 0.f;
              if (2 * c + 1 >= lim) p.y = 0.f;
            }
          } else {
            p = make_float2(ex2(xx.x), ex2(xx.y));
          }
          rs2[c & 3] = __fadd2_rn(rs2[c & 3], p);
          pk[c] = pack_bf16(p.x, p.y);
        };
        // P as bf16 pairs in columns [c0, c1) of S's region (16 at a time),
        // then the part's barrier.
        auto store_p = [&](auto c0, auto c1, uint64_t* bar) {
#pragma unroll
          for (int c = decltype(c0)::value; c < decltype(c1)::value; c += 16)
            tmem_st16(lane_base + col_s + c, *reinterpret_cast<const uint32_t(*)[16]>(&pk[c]));
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar);
        };
        static_for<kPParts>([&](auto q) {
          constexpr int Q = decltype(q)::value;
#pragma unroll
          for (int c = Q * kPCols; c < (Q + 1) * kPCols; ++c) exp_pair(c);
          if (Q == kPParts - 1) {
            const float2 rsa =
                __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
            l += rsa.x + rsa.y;
          }
          store_p(std::integral_constant<int, Q * kPCols>{},
                  std::integral_constant<int, (Q + 1) * kPCols>{}, p_full + kPParts * x + Q);
        });
      }
      // -------------------------------------------------------- epilogue
      // o_done completes once per P V of this tile; its last phase of this
      // item is s_base + n_kv - 1.
      if (ok && n_kv > 0 &&
          wait_all(o_done + x, (s_base + n_kv - 1) & 1, abort, ctl, kSiteFwdEpilogue)) {
        tc_fence_after();
        // l = 0 only for a row the block mask hides completely: O = 0.
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const bool valid = q_idx < N;
        const float lse_row = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (SPLIT) {
          float4* prw = reinterpret_cast<float4*>(sk.part_o + prow * D);
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o16[16];
            tmem_ld16(lane_base + col_o + c * 16, o16);
            tmem_wait_ld();
            if (valid)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                prw[4 * c + e] = make_float4(__uint_as_float(o16[4 * e]) * inv_l,
                                             __uint_as_float(o16[4 * e + 1]) * inv_l,
                                             __uint_as_float(o16[4 * e + 2]) * inv_l,
                                             __uint_as_float(o16[4 * e + 3]) * inv_l);
          }
          if (valid) sk.part_lse[prow] = lse_row;
        } else {
          // O rows of this warp: 64 columns per TMA store (columns past d
          // and rows past N are not written by the store).
          // This warp's staging buffer (1 KB aligned: the 128-byte swizzle
          // pattern repeats every 8 rows): row `lane`, 16-byte chunk c at
          // chunk c ^ (lane % 8) of the row.  Its previous store must have
          // read it first.
          const int row0 = qt_x * kBM + (warp & 3) * 32;
#pragma unroll
          for (int b = 0; b < C::NB; ++b) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
            const uint32_t rowa = sbase + C::STG_OFF + warp * C::STG + lane * 128;
#pragma unroll
            for (int hf = 0; hf < 4; ++hf) {  // 16 columns = 2 chunks at a time
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
          if (valid) lse[static_cast<size_t>(bh) * N + q_idx] = lse_row;
        }
        // The next item's first P V (accumulate off) overwrites O_x only
        // after this warpgroup's next P, so the loads above are complete.
        tc_fence_before();
      } else if (ok && n_kv > 0) {
        ok = false;
      }
      s_base += static_cast<uint32_t>(n_kv);
    }
    // Shared memory must outlive the O stores that read it.
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

template <int D, bool CAUSAL, bool BS, bool SPLIT>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& to, void* o, float* lse, int BH, int N, float scale,
                   const BlockMaskArg& bm, const SplitKv& sk, const Launch& L) {
  using C = Cfg<D>;
  static bool configured = false;
  if (!configured) {
    // The register split above assumes the kernel was compiled to exactly
    // kLaunchRegs per thread; with fewer, the increase would wait forever.
    cudaFuncAttributes fattr;
    cudaError_t e = cudaFuncGetAttributes(&fattr, fwd_kernel<D, CAUSAL, BS, SPLIT>);
    if (e != cudaSuccess) return e;
    if (fattr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(fwd_kernel<D, CAUSAL, BS, SPLIT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_t = (N + kBM - 1) / kBM;
  const int n_pair = (n_t + 1) / 2;
  // Heads per group: the operands every item of a head re-reads are K and V
  // (4 N_k d bytes per head); a group's K and V stay within the L2 share
  // (64 MB causal, 32 MB otherwise) while Q and O stream through.  Causal
  // launches need the large groups to keep the longest-first order global
  // enough that the last items are short ones (with 12-head groups the final
  // group's long items started last and left ~13% of the SMs idle at the end
  // of a causal N = 4096 launch).
  const long long per_head = 4LL * sk.Nk * D;
  int group = static_cast<int>(l2_group_bytes(CAUSAL) / (per_head > 0 ? per_head : 1));
  group = group < 1 ? 1 : (group > BH ? BH : group);
  const long long blocks = static_cast<long long>(BH) * n_pair * (SPLIT ? sk.n_split : 1);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const float scale_log2 = scale * 1.4426950408889634f;
  WaitCtl ctl{L.status, L.limit_ns};
  fwd_kernel<D, CAUSAL, BS, SPLIT>
      <<<static_cast<unsigned>(blocks), kThreads, C::SMEM, L.stream>>>(
          tq, tk, tv, to, static_cast<__nv_bfloat16*>(o), lse, N, BH, group, scale_log2, bm.mask,
          bm.mask_heads, bm.H, sk, ctl);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& to, void* o, float* lse, int BH, int N, float scale,
                     int causal, const BlockMaskArg* bm, const Launch& L) {
  const BlockMaskArg none{nullptr, 1, 1};
  const SplitKv dense{N, 0, 1, (N + kBN - 1) / kBN, nullptr, nullptr};
  if (bm && bm->mask)
    return causal ? launch<D, true, true, false>(tq, tk, tv, to, o, lse, BH, N, scale, *bm, dense,
                                                 L)
                  : launch<D, false, true, false>(tq, tk, tv, to, o, lse, BH, N, scale, *bm,
                                                  dense, L);
  return causal ? launch<D, true, false, false>(tq, tk, tv, to, o, lse, BH, N, scale, none, dense,
                                                L)
                : launch<D, false, false, false>(tq, tk, tv, to, o, lse, BH, N, scale, none,
                                                 dense, L);
}

template <int D>
cudaError_t launch_split_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           int BH, int Nq, float scale, int causal, const SplitKv& sk,
                           const Launch& L) {
  // Split launches write fp32 partials with plain stores: the O map is unused.
  const BlockMaskArg none{nullptr, 1, 1};
  return causal ? launch<D, true, false, true>(tq, tk, tv, tq, nullptr, nullptr, BH, Nq, scale,
                                               none, sk, L)
                : launch<D, false, false, true>(tq, tk, tv, tq, nullptr, nullptr, BH, Nq, scale,
                                                none, sk, L);
}

}  // namespace fwd

cudaError_t launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, void* o, float* lse, int BH, int N, int d,
                             float scale, int causal, const BlockMaskArg* bm, const Launch& L) {
  switch (d) {
    case 64:
      return fwd::launch_d<64>(tq, tk, tv, to, o, lse, BH, N, scale, causal, bm, L);
    case 80:
      return fwd::launch_d<80>(tq, tk, tv, to, o, lse, BH, N, scale, causal, bm, L);
    case 128:
      return fwd::launch_d<128>(tq, tk, tv, to, o, lse, BH, N, scale, causal, bm, L);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fwd_splitkv_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                     const CUtensorMap& tv, int BH, int Nq, int d, float scale,
                                     int causal, const SplitKv& sk, const Launch& L) {
  switch (d) {
    case 64:
      return fwd::launch_split_d<64>(tq, tk, tv, BH, Nq, scale, causal, sk, L);
    case 80:
      return fwd::launch_split_d<80>(tq, tk, tv, BH, Nq, scale, causal, sk, L);
    case 128:
      return fwd::launch_split_d<128>(tq, tk, tv, BH, Nq, scale, causal, sk, L);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace fa
