// fa_bwd_sm100.cu -- bf16 attention backward on B200 tensor cores (tcgen05).
//
// What it computes ("FlashAttention-2: Faster Attention with Better
// Parallelism and Work Partitioning" review page, core-algorithm answer,
// (3) backward pass; "[LLM] Flash Attention" blog, "Recomputation"):
// the softmax is recomputed tile by tile from Q, K and the saved row
// statistic instead of reading a stored S or P, and
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D),  D = rowsum(dO o O),
//   dQ = scale dS K,  dK = scale dS^T Q.
// (The page prints dS as "dP.P - P.(dP.P^T)" and drops the scale; the
// row-wise softmax Jacobian and the chain-rule scale are the reading used.)
//
// B200 design: two kernels, each parallel over batch, head and sequence (the
// FA2 review's results answer: parallelism over the sequence length), and
// each keeping every MMA operand it can in tensor memory (TMEM), because the
// shared-memory port (128 B/clk/SM) is what limits a 128 x 128 tile pair:
//
//  dK/dV kernel -- one CTA per (head, 128-key tile K_j, V_j), looping over the
//  query tiles Q_i that see it.  Per Q tile:
//      S^T  = K_j Q_i^T   (SS)  -> TMEM A = cols [0,128)
//      dP^T = V_j dO_i^T  (SS)  -> TMEM B = cols [128,256)
//      softmax warps: P^T = 2^(S^T c - LSE2) and dS^T = P^T o (dP^T - D),
//        both written (bf16) into B once dP^T has been read from it
//      dV += P^T dO_i     (TS, P^T from TMEM)  -> cols [256,256+d)
//      dK += dS^T Q_i     (TS, dS^T from TMEM) -> cols [384,384+d)
//    A only ever holds S^T: as soon as the softmax has read S^T_i into
//    registers, S^T_{i+1} is issued into A, so the tensor core computes it
//    while the softmax still works on P^T_i.  Issue order S_0, dP_0,
//    [S_0 read] S_1, [P_0] dV_0, [dS_0] dK_0, dP_1, [S_1 read] S_2, ...
//  dQ kernel -- one CTA per (head, 128-query tile Q_i), looping over the key
//  tiles K_j it sees.  Per key tile:
//      S  = Q_i K_j^T     (SS)  -> TMEM cols [0,128)
//      dP = dO_i V_j^T    (SS)  -> dP buffer j%2, cols [128,256) or [256,384)
//      softmax warps: dS = P o (dP - D), bf16, into the dP buffer it read
//      dQ += dS K_j       (TS, dS from TMEM) -> cols [384,384+d)
//    S_{j+1} is issued as soon as the softmax has read S_j, and dP_{j+1}
//    right behind it into the other buffer.  dQ is written once, in bf16, at
//    the end: no atomics and no fp32 dQ buffer, at the price of recomputing
//    S and dP (7 tile MMAs per tile pair instead of 5).
//  In both kernels dS leaves the softmax in two parts (32 of each half's 64
//  columns), each with its own barrier, so dK / dQ start on the first part;
//  the accumulators leave through row stores split by column halves between
//  the warpgroups, for d = 128 as whole 128-byte lines (an in-warp
//  transpose, store_rows_t128).
// Warp roles (both kernels, 10 warps): warps 0-3 and 4-7 are two softmax
// warpgroups splitting the 128 columns of every tile in halves (one thread
// per TMEM lane), warp 8 is the TMA producer, warp 9 the TMEM allocator and
// MMA issuer (one elected lane).  Work items run group-major (a few heads at
// a time, so their operands stay in L2), longest-first inside a group; the
// grid has one CTA per item and a running CTA takes further items by
// cancelling CTAs that have not started (cluster launch control), so the
// pipelines, barriers and TMEM carry over from item to item.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int kT = 128;  // rows of every tile (keys or queries)
// dK/dV kernel: one column pair in this many takes the FMA-pipe exp2 (0: none).
#ifndef FA_BWD_POLY_EVERY
#define FA_BWD_POLY_EVERY 0
#endif
constexpr int kBwdPolyMod = FA_BWD_POLY_EVERY > 0 ? FA_BWD_POLY_EVERY : 1;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Shape {
  static constexpr int NB = (D + 63) / 64;
  static constexpr int BLK = 64 * kT * 2;  // one 128-row x 64-col bf16 swizzle block
  static constexpr int TILE = NB * BLK;
  static constexpr int KSTEPS = D / 16;
  static_assert(D % 16 == 0 && D <= 128, "head dim must be a multiple of 16, <= 128");
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(a, parity)) {
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      atomicCAS(ctl.status, 0, kSiteBwdDrain);
      return;
    }
  }
}

// Warp-uniform bounded wait: false on every lane if any lane gave up.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort,
                                         const WaitCtl& ctl, int site) {
  const bool w = mbar_wait(bar, parity, abort, ctl, site);
  return __all_sync(0xffffffffu, w);
}

// (head, tile) of work item idx in group-major order: `group` heads at a
// time; inside a group tile index t ascending, head fastest.
__device__ __forceinline__ void group_major(int idx, int n_tiles, int BH, int group, int& bh,
                                            int& t) {
  const int per_group = group * n_tiles;
  const int g = idx / per_group;
  const int r = idx - g * per_group;
  const int gh = min(group, BH - g * group);
  t = r / gh;
  bh = g * group + (r - t * gh);
}

// Tiles visited under a block mask, as 32-tile ballot words (see TileCursor;
// all lanes of a converged warp call word()).
// ColTiles: query tiles i in [lo, n_t) whose mask byte (i, j) is set -- the
// query tiles that see key tile j (dK/dV kernel).
struct ColTiles {
  const uint8_t* m;  // [n_t][n_t] mask of the head
  int n_t, j, lo;
  __device__ __forceinline__ uint32_t word(int w) const {
    const int i = 32 * w + lane_id();
    return __ballot_sync(0xffffffffu,
                         i >= lo && i < n_t && m[static_cast<size_t>(i) * n_t + j] != 0);
  }
};
// RowTiles: key tiles j < hi whose mask byte (i, j) is set -- the key tiles
// query tile i sees (dQ kernel).
struct RowTiles {
  const uint8_t* r;  // mask row of query tile i
  int n_t, hi;
  __device__ __forceinline__ uint32_t word(int w) const {
    const int j = 32 * w + lane_id();
    return __ballot_sync(0xffffffffu, j < hi && r[j] != 0);
  }
};
template <class Tiles>
__device__ __forceinline__ int count_tiles(const Tiles& t) {
  int c = 0;
  for (int w = 0; w < (t.n_t + 31) / 32; ++w) c += __popc(t.word(w));
  return c;
}

// Store one row of a tile from TMEM columns [taddr, taddr + D) (fp32, times
// `mul`) to global memory as bf16, 16 columns (32 bytes) per step; warpgroup
// h = 0 takes the first half of the steps and h = 1 the second, so each
// 128-byte line of a row is written by one thread (measured: +0.3 % backward
// at N = 4096, +1.1 % at N = 512 over alternating steps).  Every thread
// writes its own row, so a warp's store touches 32 rows: with `wide` (the
// tensor 32-byte aligned, hence every 32-byte piece of a row) each piece is
// one 32-byte store, a whole L2 sector, instead of two 16-byte halves.
template <int D>
__device__ __forceinline__ void store_row_bf16(uint32_t taddr, float mul, __nv_bfloat16* row,
                                               bool valid, int h, bool wide) {
#pragma unroll
  for (int c = 0; c < D / 16; ++c) {
    if ((2 * c >= D / 16) != (h == 1)) continue;  // h = 0: the first half of the chunks
    uint32_t v16[16];
    tmem_ld16(taddr + c * 16, v16);
    tmem_wait_ld();
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      pk[e] = pack_bf16(__uint_as_float(v16[2 * e]) * mul, __uint_as_float(v16[2 * e + 1]) * mul);
    if (valid) {
      if (wide) {
        st_global_v8(row + c * 16, pk);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(row + c * 16);
        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
  }
}

// The same for d = 128 with whole 128-byte lines per store: this warp's 32
// rows, columns [64 h, 64 h + 64) (128 bytes of each row), from TMEM
// (thread t holds row t), packed to bf16 in 16-byte pieces.  Within each
// group of 8 lanes an 8 x 8 transpose of the pieces (three butterfly stages
// of shuffles: at stage m a lane swaps with lane ^ m the pieces whose index
// bit m differs from its own lane bit m) leaves lane 8 g + s holding piece s
// of rows 8 g + 0..7; store k then writes rows 8 g + k for g = 0..3, four
// whole lines, where the row-per-lane store writes 32 pieces of 32 rows
// (8x fewer L2 write requests).  Rows at or past n_valid are not written.
__device__ __forceinline__ void store_rows_t128(uint32_t taddr, float mul,
                                                __nv_bfloat16* warp_row0, int n_valid, int h,
                                                int lane) {
  uint32_t t0[32], t1[32];
  tmem_ld32(taddr + 64 * h, t0);
  tmem_ld32(taddr + 64 * h + 32, t1);
  tmem_wait_ld();
  uint32_t e[8][4];  // piece c: columns 64 h + 8 c .. + 8 of this thread's row
#pragma unroll
  for (int c = 0; c < 8; ++c)
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = 8 * c + 2 * w;  // column within the half
      const float a = __uint_as_float(j < 32 ? t0[j] : t1[j - 32]);
      const float b = __uint_as_float(j + 1 < 32 ? t0[j + 1] : t1[j + 1 - 32]);
      e[c][w] = pack_bf16(a * mul, b * mul);
    }
  const int sub = lane & 7;
#pragma unroll
  for (int m = 4; m >= 1; m >>= 1) {
    const bool up = (sub & m) != 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c & m) continue;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t send = up ? e[c][w] : e[c ^ m][w];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
        if (up)
          e[c][w] = recv;
        else
          e[c ^ m][w] = recv;
      }
    }
  }
  const int g = lane >> 3;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = 8 * g + k;
    if (r < n_valid)
      *reinterpret_cast<uint4*>(warp_row0 + static_cast<size_t>(r) * 128 + 64 * h + 8 * sub) =
          make_uint4(e[k][0], e[k][1], e[k][2], e[k][3]);
  }
}

// P^T of one key row (64 queries of a half tile): 2^(S^T c - LSE2[q]) from
// the S^T values `sv` and the staged LSE2 vector `l2`, packed to bf16 pairs.
// MASK zeroes queries q < qlo (diagonal tile, key past N); the unmasked
// instantiation, used by every tile a whole warp sees unmasked, has no
// selects in the loop.
template <bool MASK>
__device__ __forceinline__ void kv_p_row(const uint32_t (&sv)[2][32], const float* l2, float2 sc2,
                                         int qlo, uint32_t (&pk)[32]) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const float4 lv = *reinterpret_cast<const float4*>(l2 + c * 32 + e);
      const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sv[c][e]),
                                                __uint_as_float(sv[c][e + 1])),
                                    sc2, make_float2(-lv.x, -lv.y));
      const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sv[c][e + 2]),
                                                __uint_as_float(sv[c][e + 3])),
                                    sc2, make_float2(-lv.z, -lv.w));
      // one pair in FA_BWD_POLY_EVERY on the FMA pipe, the rest on the MUFU
      float2 p01, p23;
      if (FA_BWD_POLY_EVERY > 0 && ((c * 16 + e / 2) % kBwdPolyMod) == kBwdPolyMod - 1)
        p01 = exp2_fma2(x01);
      else
        p01 = make_float2(ex2(x01.x), ex2(x01.y));
      if (FA_BWD_POLY_EVERY > 0 && ((c * 16 + e / 2 + 1) % kBwdPolyMod) == kBwdPolyMod - 1)
        p23 = exp2_fma2(x23);
      else
        p23 = make_float2(ex2(x23.x), ex2(x23.y));
      if (MASK) {
        const int q0 = c * 32 + e;  // query within this half
        if (q0 + 0 < qlo) p01.x = 0.f;
        if (q0 + 1 < qlo) p01.y = 0.f;
        if (q0 + 2 < qlo) p23.x = 0.f;
        if (q0 + 3 < qlo) p23.y = 0.f;
      }
      pk[c * 16 + e / 2] = pack_bf16(p01.x, p01.y);
      pk[c * 16 + e / 2 + 1] = pack_bf16(p23.x, p23.y);
    }
  }
}

// P of one query row (64 keys of a half tile) in the dQ kernel:
// 2^(S c - LSE2) for keys c < lim, 0 past it (MASK); unmasked rows take the
// select-free instantiation.
template <bool MASK>
__device__ __forceinline__ void dq_p_row(const uint32_t (&sv)[2][32], float scale_log2,
                                         float my_l2, int lim, float (&p)[64]) {
  const float2 sc2 = make_float2(scale_log2, scale_log2);
  const float2 nl2 = make_float2(-my_l2, -my_l2);
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[c >> 5][c & 31]),
                                            __uint_as_float(sv[c >> 5][(c & 31) + 1])),
                                sc2, nl2);
    p[c] = ex2(x.x);
    p[c + 1] = ex2(x.y);
    if (MASK) {
      if (c >= lim) p[c] = 0.f;
      if (c + 1 >= lim) p[c + 1] = 0.f;
    }
  }
}

// =========================================================================
// dK / dV
// =========================================================================

template <int D>
struct KvCfg : Shape<D> {
  using S = Shape<D>;
  // S^T_{i+1} is issued as soon as the softmax has read S^T_i, about one
  // iteration before dK_i releases Q_i's stage: Q needs three stages so that
  // Q_{i+1} has landed by then.  dO_i is released by dV_i and first needed
  // by dP_i at the end of iteration i - 1: two stages suffice.
  static constexpr int NQ = 3, NDO = 2;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + S::TILE;
  static constexpr int Q_OFF = V_OFF + S::TILE;          // [NQ] stages
  static constexpr int DO_OFF = Q_OFF + NQ * S::TILE;    // [NDO] stages
  static constexpr int LSE_OFF = DO_OFF + NDO * S::TILE; // [NQ] x 512 B: the Q tile's LSE2
  static constexpr int DV_OFF = LSE_OFF + NQ * 512;      // [NDO] x 512 B: the dO tile's D
  static constexpr int BAR_OFF = DV_OFF + NDO * 512;
  static constexpr int NBAR = 24;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // 16-byte aligned (next-item responses)
  static constexpr int USED = MISC_OFF + 48;
  // Slack for aligning the dynamic shared memory to 1 KB, as far as the
  // budget allows; the kernel checks at run time that it was enough.
  static constexpr int SLACK = USED + 1024 <= 232448 ? 1024 : 232448 - USED;
  static constexpr int SMEM = USED + SLACK;
  static_assert(MISC_OFF % 16 == 0, "next-item responses need 16-byte alignment");
  static_assert(SLACK >= 0 && SMEM <= 232448, "shared memory budget");
};

// TMEM columns of the dK/dV kernel.  Region A holds S^T only, region B dP^T
// and then the softmax results: warpgroup h reads S^T columns [64h, 64h+64)
// of A and dP^T columns [128+64h, +64) of B, then writes its P^T (bf16
// pairs) into [128+64h, +32) and its dS^T into [128+64h+32, +32).
constexpr uint32_t kKvColS = 0, kKvColDP = 128, kKvColDV = 256, kKvColDK = 384;
constexpr uint32_t kKvOffP = 0, kKvOffDS = 32;  // within a warpgroup's 64 columns of B

template <int D, bool CAUSAL, bool BS>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ dvec,
                    const float* __restrict__ lse2, __nv_bfloat16* __restrict__ dk,
                    __nv_bfloat16* __restrict__ dv, int N, int BH, int group, float scale,
                    float scale_log2, const uint8_t* __restrict__ bmask, int mask_heads, int H,
                    bool wide, WaitCtl ctl) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  {
    // The budget may leave less than 1 KB of alignment slack (d = 80, 128):
    // give up, recorded in the status word, if the base needs more.
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad > static_cast<uint32_t>(C::SLACK)) {
      if (threadIdx.x == 0) atomicCAS(ctl.status, 0, kSiteBwdSmem);
      return;
    }
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;     // [NQ]  Q_i and its LSE2
  uint64_t* q_empty = bars + 4;    // [NQ]  dK_i is done with Q_i
  uint64_t* do_full = bars + 7;    // [NDO] dO_i and its D
  uint64_t* do_empty = bars + 9;   // [NDO] dV_i is done with dO_i
  uint64_t* s_full = bars + 11;
  uint64_t* dp_full = bars + 12;
  uint64_t* p_full = bars + 13;    // both softmax warpgroups wrote P^T
  uint64_t* ds_full = bars + 14;   // both wrote dS^T, queries [0, 32) of each half
  uint64_t* kv_done = bars + 15;   // the item's last dK: accumulators final
  uint64_t* kv_empty = bars + 16;  // the item's S^T and dP^T MMAs are done with K_j, V_j
  uint64_t* nxt_full = bars + 17;  // [2] next-item requests
  uint64_t* nxt_empty = bars + 19; // [2]
  uint64_t* s_read = bars + 21;    // both softmax warpgroups have S^T in registers
  uint64_t* ds_full2 = bars + 22;  // both wrote dS^T, queries [32, 64) of each half
  uint8_t* nxt_resp = smem + C::MISC_OFF;  // [2] x 16 bytes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF + 32);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 36);

  const int warp = warp_id();
  const int lane = lane_id();
  const int n_t = (N + kT - 1) / kT;
  const int Np = n_t * kT;
  // Key tile j and the query tiles [i_start, n_t) that see it, for work item
  // idx (group-major; j = 0 first: most query tiles when causal).
  // With a block mask (BS) only the query tiles whose mask byte (i, j) is set
  // are visited (`tiles`, walked with a TileCursor).  Every role calls this
  // with its whole (converged) warp.
  ColTiles tiles{bmask, n_t, 0, 0};
  auto decode = [&](int idx, int& bh, int& j, int& i_start, int& n_iter) {
    group_major(idx, n_t, BH, group, bh, j);
    i_start = CAUSAL ? j : 0;
    n_iter = n_t - i_start;
    if (BS) {
      tiles = ColTiles{bmask + static_cast<size_t>(mask_heads == 1 ? 0 : bh % H) * n_t * n_t,
                       n_t, j, i_start};
      n_iter = count_tiles(tiles);
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < C::NQ; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    for (int s = 0; s < C::NDO; ++s) {
      mbar_init(do_full + s, 1);
      mbar_init(do_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(nxt_full + s, 1);
      mbar_init(nxt_empty + s, 9);  // MMA warp + 8 softmax warps
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    // softmax-side barriers: one arrival per softmax warp
    mbar_init(s_read, 8);
    mbar_init(p_full, 8);
    mbar_init(ds_full, 8);
    mbar_init(ds_full2, 8);
    mbar_init(kv_done, 1);
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
  auto next_item = [&](int it, int& idx, int site) -> bool {
    return next_work_item(it, idx, nxt_full, nxt_empty, nxt_resp, abort, ctl, site);
  };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop (it reads the block mask with all lanes);
    // the elected lane issues the copies and the next-item requests.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
    }
    int last_q[C::NQ], last_do[C::NDO];  // last ring use of each stage (drained on abort)
#pragma unroll
    for (int s = 0; s < C::NQ; ++s) last_q[s] = -1;
#pragma unroll
    for (int s = 0; s < C::NDO; ++s) last_do[s] = -1;
    int kv_issued = 0;
    int nxt_pending = -1;
    uint32_t nxt_pending_par = 0;
    uint32_t qr = 0;  // query tiles streamed so far (ring uses)
    int idx = static_cast<int>(blockIdx.x);
    bool ok = true;
    for (int w = 0; ok; ++w) {
      if (w > 0) {
        if (!producer_take_item(w, idx, nxt_full, nxt_resp, abort, ctl, kSiteBwdProducer)) break;
        nxt_pending = -1;
        if (idx < 0) break;
      }
      // Ask for item w + 1 right away, so its loads can follow this item's.
      if (!producer_request_item(w, nxt_full, nxt_empty, nxt_resp, abort, ctl, kSiteBwdProducer,
                                 leader, nxt_pending, nxt_pending_par))
        break;
      int bh, j, i_start, n_iter;
      decode(idx, bh, j, i_start, n_iter);
      if (n_iter > 0) {
        if (kv_issued > 0 && !wait_all(kv_empty, static_cast<uint32_t>(kv_issued - 1) & 1, abort,
                                       ctl, kSiteBwdProducer))
          break;
        if (leader) {
          mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
#pragma unroll
          for (int b = 0; b < C::NB; ++b) {
            tma_load_3d(&tm_k, kv_full, smem + C::K_OFF + b * C::BLK, b * 64, j * kT, bh);
            tma_load_3d(&tm_v, kv_full, smem + C::V_OFF + b * C::BLK, b * 64, j * kT, bh);
          }
        }
        __syncwarp();
        ++kv_issued;
        TileCursor cur(n_t);
        for (int it = 0; it < n_iter; ++it, ++qr) {
          const int ic = BS ? cur.next(tiles) : i_start + it;  // query tile of the step
          const int y = ic * kT;
          const size_t vrow = static_cast<size_t>(bh) * Np + y;
          const int sq = static_cast<int>(qr % C::NQ), sd = static_cast<int>(qr % C::NDO);
          const uint32_t uq = qr / C::NQ, ud = qr / C::NDO;
          if (qr >= C::NQ && !wait_all(q_empty + sq, (uq - 1) & 1, abort, ctl, kSiteBwdProducer)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(q_full + sq, C::TILE + 512);
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
              tma_load_3d(&tm_q, q_full + sq, smem + C::Q_OFF + sq * C::TILE + b * C::BLK,
                          b * 64, y, bh);
            bulk_load_1d(smem + C::LSE_OFF + sq * 512, lse2 + vrow, 512, q_full + sq);
          }
          __syncwarp();
          last_q[sq] = static_cast<int>(uq);
          if (qr >= C::NDO &&
              !wait_all(do_empty + sd, (ud - 1) & 1, abort, ctl, kSiteBwdProducer)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(do_full + sd, C::TILE + 512);
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
              tma_load_3d(&tm_do, do_full + sd, smem + C::DO_OFF + sd * C::TILE + b * C::BLK,
                          b * 64, y, bh);
            bulk_load_1d(smem + C::DV_OFF + sd * 512, dvec + vrow, 512, do_full + sd);
          }
          __syncwarp();
          last_do[sd] = static_cast<int>(ud);
        }
        if (!ok) break;
      }
    }
    if (*abort && leader) {
      if (kv_issued > 0) drain_wait(kv_full, static_cast<uint32_t>(kv_issued - 1) & 1, ctl);
      for (int s = 0; s < C::NQ; ++s)
        if (last_q[s] >= 0) drain_wait(q_full + s, last_q[s] & 1, ctl);
      for (int s = 0; s < C::NDO; ++s)
        if (last_do[s] >= 0) drain_wait(do_full + s, last_do[s] & 1, ctl);
      if (nxt_pending >= 0) drain_wait(nxt_full + nxt_pending, nxt_pending_par, ctl);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    // All lanes run the schedule; the elected lane issues MMAs and commits.
    const bool leader = elect_one();
    constexpr uint32_t kIdescSq = idesc_bf16(kT, kT, 0, 0);  // S^T, dP^T
    constexpr uint32_t kIdescAcc = idesc_bf16(kT, D, 0, 1);  // dV, dK (B MN-major)
    const SDesc k_desc = sdesc(sbase + C::K_OFF, 16, 1024);           // K-major (A)
    const SDesc v_desc = sdesc(sbase + C::V_OFF, 16, 1024);           // K-major (A)
    const SDesc q_desc = sdesc(sbase + C::Q_OFF, 16, 1024);           // K-major (B of S^T)
    const SDesc do_desc = sdesc(sbase + C::DO_OFF, 16, 1024);         // K-major (B of dP^T)
    const SDesc q_mn = sdesc(sbase + C::Q_OFF, C::BLK, 1024);         // MN-major (B of dK)
    const SDesc do_mn = sdesc(sbase + C::DO_OFF, C::BLK, 1024);       // MN-major (B of dV)
    uint32_t qbase = 0;  // query tiles of the previous items (ring uses, barrier phases)
    int n_iter = 0, s_done = 0, dp_done = 0, released = 0;
    auto release_kv = [&]() {  // after the item's last S^T and dP^T
      if (!released && s_done == n_iter && dp_done == n_iter) {
        if (leader) mma_commit(kv_empty);
        __syncwarp();
        released = 1;
      }
    };
    auto issue_s = [&](int it) -> bool {  // S^T = K_j Q_i^T -> region A
      const uint32_t g = qbase + it;
      const int sq = static_cast<int>(g % C::NQ);
      if (!wait_all(q_full + sq, (g / C::NQ) & 1, abort, ctl, kSiteBwdMma)) return false;
      tc_fence_after();
      if (leader) {
        const SDesc qd = q_desc + sq * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + kKvColS, k_desc + off, qd + off, kIdescSq, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
      }
      __syncwarp();
      ++s_done;
      release_kv();
      return true;
    };
    auto issue_dp = [&](int it) -> bool {  // dP^T = V_j dO_i^T -> region B
      const uint32_t g = qbase + it;
      const int sd = static_cast<int>(g % C::NDO);
      if (!wait_all(do_full + sd, (g / C::NDO) & 1, abort, ctl, kSiteBwdMma)) return false;
      tc_fence_after();
      if (leader) {
        const SDesc dd = do_desc + sd * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + kKvColDP, v_desc + off, dd + off, kIdescSq, kk > 0 ? 1u : 0u);
        }
        mma_commit(dp_full);
      }
      __syncwarp();
      ++dp_done;
      release_kv();
      return true;
    };
    // S^T_{i+1} overwrites S^T_i in A once both warpgroups have read it
    // (s_read).  dP^T_{i+1} overwrites P^T_i and dS^T_i in B: issued after
    // dV_i and dK_i (same thread, in order), which read them.
    bool ok = true;
    int idx = 0;
    uint32_t kv_items = 0;  // items with at least one query tile (one K/V load each)
    for (int w = 0; ok; ++w) {
      if (!next_item(w, idx, kSiteBwdMma)) break;
      if (idx < 0) break;
      int bh, j, i_start;
      decode(idx, bh, j, i_start, n_iter);
      if (n_iter == 0) continue;  // the block mask hides this key tile from every query
      s_done = dp_done = released = 0;
      ok = wait_all(kv_full, kv_items & 1, abort, ctl, kSiteBwdMma) && issue_s(0) &&
           issue_dp(0);
      ++kv_items;
      for (int it = 0; ok && it < n_iter; ++it) {
        const uint32_t g = qbase + it;
        const int sq = static_cast<int>(g % C::NQ), sd = static_cast<int>(g % C::NDO);
        const SDesc qm = q_mn + sq * C::TILE;
        const SDesc dm = do_mn + sd * C::TILE;
        if (it + 1 < n_iter) {
          if (!wait_all(s_read, g & 1, abort, ctl, kSiteBwdMma) || !issue_s(it + 1)) {
            ok = false;
            break;
          }
        }
        // dV += P^T dO_i: query k-step kk (16 queries) lives in columns
        // 64*(kk/4) + 8*(kk%4) of the P^T half of B.
        if (!wait_all(p_full, g & 1, abort, ctl, kSiteBwdMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)
            mma_ts(tmem + kKvColDV, tmem + kKvColDP + kKvOffP + (kk >> 2) * 64 + (kk & 3) * 8,
                   dm + kk * 2048, kIdescAcc,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(do_empty + sd);
        }
        __syncwarp();
        // dK += dS^T Q_i: dS^T k-step kk at column 64*(kk/4) + 8*(kk%4) of
        // the dS^T half of B.  dS^T arrives in two parts (k-steps with
        // kk%4 < 2, then the rest), and each part's MMAs go as soon as it is in.
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          if (!wait_all(part ? ds_full2 : ds_full, g & 1, abort, ctl, kSiteBwdMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kh = 0; kh < 2; ++kh)
#pragma unroll
              for (int k2 = 0; k2 < 2; ++k2) {
                const int kk = 4 * kh + 2 * part + k2;
                mma_ts(tmem + kKvColDK,
                       tmem + kKvColDP + kKvOffDS + (kk >> 2) * 64 + (kk & 3) * 8,
                       qm + kk * 2048, kIdescAcc, (it > 0 || kk > 0) ? 1u : 0u);
              }
            if (part) mma_commit(q_empty + sq);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (it + 1 < n_iter && !issue_dp(it + 1)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (leader) mma_commit(kv_done);
      __syncwarp();
      qbase += static_cast<uint32_t>(n_iter);
    }
    __syncwarp();
  } else {
    // ------------------------- P^T and dS^T (warps 0-3: queries 0-63, 4-7: 64-127)
    const int h = warp >> 2;
    const int kr = threadIdx.x & 127;  // key row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t col_s = kKvColS + 64 * h;    // this half's S^T
    const uint32_t col_dp = kKvColDP + 64 * h;  // this half's dP^T, then P^T and dS^T
    uint32_t qbase = 0;     // query tiles of the previous items (barrier phases)
    uint32_t kv_items = 0;  // items with at least one query tile
    bool ok = true;
    int idx = 0;
    // One arrival per warp once every lane's tcgen05 loads / stores are done.
    auto warp_arrive = [&](uint64_t* bar) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    for (int w = 0; ok; ++w) {
      if (!next_item(w, idx, kSiteBwdSoftmax)) break;
      if (idx < 0) break;
      int bh, j, i_start, n_iter;
      decode(idx, bh, j, i_start, n_iter);
      const int k_idx = j * kT + kr;
      const bool key_ok = k_idx < N;
      if (n_iter == 0) {
        // No query sees this key tile: dK = dV = 0 (block mask only).
        const size_t row = (static_cast<size_t>(bh) * N + k_idx) * D;
        if (key_ok)
          for (int c = h; c < D / 8; c += 2) {
            reinterpret_cast<uint4*>(dv + row)[c] = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4*>(dk + row)[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        continue;
      }
      TileCursor cur(n_t);
      for (int it = 0; it < n_iter; ++it) {
        const int i = BS ? cur.next(tiles) : i_start + it;  // query tile of the step
        const uint32_t g = qbase + it;
        // LSE2 and D of this half's 64 queries, staged by the producer with
        // the Q tile (q_full completed before S^T, hence before s_full) and
        // the dO tile (do_full completed before dP^T, hence before dp_full).
        const float* l2 =
            reinterpret_cast<const float*>(smem + C::LSE_OFF + (g % C::NQ) * 512) + 64 * h;
        const float* dd =
            reinterpret_cast<const float*>(smem + C::DV_OFF + (g % C::NDO) * 512) + 64 * h;
        const bool diag = CAUSAL && (i == j);
        if (!wait_all(s_full, g & 1, abort, ctl, kSiteBwdSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[2][32];
        tmem_ld32(lane_base + col_s, sv[0]);
        tmem_ld32(lane_base + col_s + 32, sv[1]);
        tmem_wait_ld();
        warp_arrive(s_read);  // A may take S^T_{i+1} now
        const float2 sc2 = make_float2(scale_log2, scale_log2);
        // queries of this half this key row sees: all, none (key past N), or
        // q >= key on the diagonal tile
        const int qlo = !key_ok ? 64 : (diag ? kr - 64 * h : 0);
        uint32_t pk[32];  // P^T of this half, bf16 pairs
        if (__any_sync(0xffffffffu, qlo > 0))
          kv_p_row<true>(sv, l2, sc2, qlo, pk);
        else
          kv_p_row<false>(sv, l2, sc2, qlo, pk);

        if (!wait_all(dp_full, g & 1, abort, ctl, kSiteBwdSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t dpv[2][32];
        tmem_ld32(lane_base + col_dp, dpv[0]);
        tmem_ld32(lane_base + col_dp + 32, dpv[1]);
        tmem_wait_ld();
        // P^T -> the first 32 of this half's dP^T columns (just read).
        tmem_st32(lane_base + col_dp + kKvOffP, pk);
        tmem_wait_st();
        warp_arrive(p_full);
        // dS^T = P^T o (dP^T - D), formed as P dP - P D on column pairs
        // (two paired fp32 operations per pair).  Each 32-query part goes
        // to the last 32 of this half's dP^T columns as soon as it is formed.
        uint32_t dsk[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 dv4 = *reinterpret_cast<const float4*>(dd + c * 32 + e);
            const uint32_t p01 = pk[c * 16 + e / 2], p23 = pk[c * 16 + e / 2 + 1];
            const float2 pa = make_float2(bf16lo(p01), bf16hi(p01));
            const float2 pb = make_float2(bf16lo(p23), bf16hi(p23));
            const float2 ra = __ffma2_rn(pa, make_float2(__uint_as_float(dpv[c][e + 0]),
                                                         __uint_as_float(dpv[c][e + 1])),
                                         __fmul2_rn(pa, make_float2(-dv4.x, -dv4.y)));
            const float2 rb = __ffma2_rn(pb, make_float2(__uint_as_float(dpv[c][e + 2]),
                                                         __uint_as_float(dpv[c][e + 3])),
                                         __fmul2_rn(pb, make_float2(-dv4.z, -dv4.w)));
            dsk[c * 16 + e / 2] = pack_bf16(ra.x, ra.y);
            dsk[c * 16 + e / 2 + 1] = pack_bf16(rb.x, rb.y);
          }
          tmem_st16(lane_base + col_dp + kKvOffDS + 16 * c,
                    *reinterpret_cast<const uint32_t(*)[16]>(&dsk[16 * c]));
          tmem_wait_st();
          warp_arrive(c ? ds_full2 : ds_full);
        }
      }
      if (!ok) break;
      // Epilogue: dV (unscaled) and dK (times scale), each warpgroup half of
      // the columns.  kv_done completes once per item; the
      // next item's first dV/dK MMAs (accumulate off) come after this
      // warpgroup's next P^T / dS^T, so the loads below are complete by then.
      if (!wait_all(kv_done, kv_items & 1, abort, ctl, kSiteBwdEpilogue)) break;
      ++kv_items;
      tc_fence_after();
      if constexpr (D == 128) {
        const int r0 = j * kT + (warp & 3) * 32;  // first key row of this warp
        const size_t w0 = (static_cast<size_t>(bh) * N + r0) * D;
        const int nv = min(max(N - r0, 0), 32);
        store_rows_t128(lane_base + kKvColDV, 1.f, dv + w0, nv, h, lane);
        store_rows_t128(lane_base + kKvColDK, scale, dk + w0, nv, h, lane);
      } else {
        const size_t row = (static_cast<size_t>(bh) * N + k_idx) * D;
        store_row_bf16<D>(lane_base + kKvColDV, 1.f, dv + row, key_ok, h, wide);
        store_row_bf16<D>(lane_base + kKvColDK, scale, dk + row, key_ok, h, wide);
      }
      tc_fence_before();
      qbase += static_cast<uint32_t>(n_iter);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// =========================================================================
// dQ
// =========================================================================

template <int D>
struct QCfg : Shape<D> {
  using S = Shape<D>;
  // K_j is used by S_j and dQ_j (late), V_j only by dP_j (early), so the K
  // ring is one stage deeper: K_{j+2} can land while dQ_j still reads K_j.
  static constexpr int NK = S::NB == 1 ? 4 : 3;
  static constexpr int NV = S::NB == 1 ? 4 : 2;
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = Q_OFF + S::TILE;
  static constexpr int K_OFF = DO_OFF + S::TILE;      // [NK]
  static constexpr int V_OFF = K_OFF + NK * S::TILE;  // [NV]
  static constexpr int BAR_OFF = V_OFF + NV * S::TILE;
  static constexpr int NBAR = (15 + 2 * NK + 2 * NV + 1) & ~1;  // even: keeps MISC 16-byte aligned
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // 16-byte aligned (next-item responses)
  static constexpr int SMEM = MISC_OFF + 48 + 1024;
  static_assert(MISC_OFF % 16 == 0, "next-item responses need 16-byte alignment");
  static_assert(SMEM <= 232448, "shared memory budget");
};

// TMEM columns of the dQ kernel: S, two dP buffers, dQ accumulator.
// Softmax warpgroup h reads S columns [64h, 64h+64) and dP columns
// [64h, 64h+64) of the current dP buffer, and writes its dS (bf16 pairs) into
// [64h, 64h+32) of that dP buffer.
constexpr uint32_t kQColS = 0, kQColDP = 128, kQColDQ = 384;

template <int D, bool CAUSAL, bool BS>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ dvec,
                  const float* __restrict__ lse2, __nv_bfloat16* __restrict__ dq, int N, int BH,
                  int group, float scale, float scale_log2, const uint8_t* __restrict__ bmask,
                  int mask_heads, int H, bool wide, WaitCtl ctl) {
  using C = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars + 0;   // Q_i and dO_i
  uint64_t* q_empty = bars + 1;  // the item's S and dP MMAs are done with Q_i, dO_i
  uint64_t* dq_done = bars + 2;
  uint64_t* k_full = bars + 3;          // [NK]
  uint64_t* k_empty = k_full + C::NK;   // [NK]
  uint64_t* v_full = k_empty + C::NK;   // [NV]
  uint64_t* v_empty = v_full + C::NV;   // [NV]
  uint64_t* s_full = v_empty + C::NV;
  uint64_t* s_read = s_full + 1;        // both softmax warpgroups have S in registers
  uint64_t* dp_full = s_read + 1;       // [2] per dP buffer
  uint64_t* ds_full = dp_full + 2;      // [2 dP buffers][2 parts: keys 0-31, 32-63 of each half]
  uint64_t* nxt_full = ds_full + 4;     // [2] next-item requests
  uint64_t* nxt_empty = nxt_full + 2;   // [2]
  uint8_t* nxt_resp = smem + C::MISC_OFF;  // [2] x 16 bytes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF + 32);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 36);

  const int warp = warp_id();
  const int lane = lane_id();
  const int n_t = (N + kT - 1) / kT;
  const int Np = n_t * kT;
  // Query tile i and the key tiles it sees for work item idx (group-major,
  // longest query tiles first when causal).
  // With a block mask (BS) only the key tiles whose mask byte (i, j) is set
  // are visited (`tiles`, walked with a TileCursor).  Every role calls this
  // with its whole (converged) warp.
  RowTiles tiles{bmask, n_t, 0};
  auto decode = [&](int idx, int& bh, int& i, int& n_kv) {
    int t;
    group_major(idx, n_t, BH, group, bh, t);
    i = n_t - 1 - t;
    n_kv = CAUSAL ? i + 1 : n_t;
    if (BS) {
      tiles = RowTiles{bmask + (static_cast<size_t>(mask_heads == 1 ? 0 : bh % H) * n_t + i) * n_t,
                       n_t, n_kv};
      n_kv = count_tiles(tiles);
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(dq_done, 1);
    for (int s = 0; s < C::NK; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(dp_full + b, 1);
      mbar_init(ds_full + 2 * b, 8);      // one arrival per softmax warp
      mbar_init(ds_full + 2 * b + 1, 8);
      mbar_init(nxt_full + b, 1);
      mbar_init(nxt_empty + b, 9);  // MMA warp + 8 softmax warps
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 8);
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
  auto next_item = [&](int it, int& idx, int site) -> bool {
    return next_work_item(it, idx, nxt_full, nxt_empty, nxt_resp, abort, ctl, site);
  };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop (it reads the block mask with all lanes);
    // the elected lane issues the copies and the next-item requests.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
    }
    int last_k[C::NK], last_v[C::NV];
#pragma unroll
    for (int s = 0; s < C::NK; ++s) last_k[s] = -1;
#pragma unroll
    for (int s = 0; s < C::NV; ++s) last_v[s] = -1;
    int q_issued = 0;
    int nxt_pending = -1;
    uint32_t nxt_pending_par = 0;
    uint32_t kr = 0;  // key tiles streamed so far (ring uses of both rings)
    int idx = static_cast<int>(blockIdx.x);
    bool ok = true;
    for (int it = 0; ok; ++it) {
      if (it > 0) {
        if (!producer_take_item(it, idx, nxt_full, nxt_resp, abort, ctl, kSiteBwdProducer)) break;
        nxt_pending = -1;
        if (idx < 0) break;
      }
      // Ask for item it + 1 right away, so its loads can follow this item's.
      if (!producer_request_item(it, nxt_full, nxt_empty, nxt_resp, abort, ctl, kSiteBwdProducer,
                                 leader, nxt_pending, nxt_pending_par))
        break;
      int bh, i, n_kv;
      decode(idx, bh, i, n_kv);
      if (n_kv > 0) {
        if (q_issued > 0 && !wait_all(q_empty, static_cast<uint32_t>(q_issued - 1) & 1, abort,
                                      ctl, kSiteBwdProducer))
          break;
        if (leader) {
          mbar_arrive_expect_tx(q_full, 2 * C::TILE);
#pragma unroll
          for (int b = 0; b < C::NB; ++b) {
            tma_load_3d(&tm_q, q_full, smem + C::Q_OFF + b * C::BLK, b * 64, i * kT, bh);
            tma_load_3d(&tm_do, q_full, smem + C::DO_OFF + b * C::BLK, b * 64, i * kT, bh);
          }
        }
        __syncwarp();
        ++q_issued;
        TileCursor cur(n_t);
        for (int jj = 0; jj < n_kv; ++jj, ++kr) {
          const int jt = BS ? cur.next(tiles) : jj;  // key tile of the step
          const int sk = static_cast<int>(kr % C::NK), sv = static_cast<int>(kr % C::NV);
          const uint32_t uk = kr / C::NK, uv = kr / C::NV;
          if (kr >= C::NK && !wait_all(k_empty + sk, (uk - 1) & 1, abort, ctl, kSiteBwdProducer)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(k_full + sk, C::TILE);
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
              tma_load_3d(&tm_k, k_full + sk, smem + C::K_OFF + sk * C::TILE + b * C::BLK, b * 64,
                          jt * kT, bh);
          }
          __syncwarp();
          last_k[sk] = static_cast<int>(uk);
          if (kr >= C::NV && !wait_all(v_empty + sv, (uv - 1) & 1, abort, ctl, kSiteBwdProducer)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(v_full + sv, C::TILE);
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
              tma_load_3d(&tm_v, v_full + sv, smem + C::V_OFF + sv * C::TILE + b * C::BLK, b * 64,
                          jt * kT, bh);
          }
          __syncwarp();
          last_v[sv] = static_cast<int>(uv);
        }
        if (!ok) break;
      }
    }
    if (*abort && leader) {
      if (q_issued > 0) drain_wait(q_full, static_cast<uint32_t>(q_issued - 1) & 1, ctl);
      for (int s = 0; s < C::NK; ++s)
        if (last_k[s] >= 0) drain_wait(k_full + s, last_k[s] & 1, ctl);
      for (int s = 0; s < C::NV; ++s)
        if (last_v[s] >= 0) drain_wait(v_full + s, last_v[s] & 1, ctl);
      if (nxt_pending >= 0) drain_wait(nxt_full + nxt_pending, nxt_pending_par, ctl);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    // All lanes run the schedule; the elected lane issues MMAs and commits.
    const bool leader = elect_one();
    constexpr uint32_t kIdescSq = idesc_bf16(kT, kT, 0, 0);  // S, dP
    constexpr uint32_t kIdescDq = idesc_bf16(kT, D, 0, 1);   // dQ (B = K_j MN-major)
    const SDesc q_desc = sdesc(sbase + C::Q_OFF, 16, 1024);     // K-major (A of S)
    const SDesc do_desc = sdesc(sbase + C::DO_OFF, 16, 1024);   // K-major (A of dP)
    const SDesc k_desc = sdesc(sbase + C::K_OFF, 16, 1024);     // K-major (B of S)
    const SDesc v_desc = sdesc(sbase + C::V_OFF, 16, 1024);     // K-major (B of dP)
    const SDesc k_mn = sdesc(sbase + C::K_OFF, C::BLK, 1024);   // MN-major (B of dQ)
    // Running counts across items: key tiles (ring uses) before this item,
    // which also number the dP buffers (buffer g & 1 for the g-th dP).
    uint32_t kbase = 0;
    int n_kv = 0, released = 0, s_done = 0, dp_done = 0;
    auto release_q = [&]() {  // after the item's last S and dP
      if (!released && s_done == n_kv && dp_done == n_kv) {
        if (leader) mma_commit(q_empty);
        __syncwarp();
        released = 1;
      }
    };
    auto issue_s = [&](int jj) -> bool {  // S_jj = Q K_jj^T -> S columns
      const uint32_t g = kbase + jj;
      const int s = static_cast<int>(g % C::NK);
      if (!wait_all(k_full + s, (g / C::NK) & 1, abort, ctl, kSiteBwdMma)) return false;
      tc_fence_after();
      if (leader) {
        const SDesc kd = k_desc + s * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + kQColS, q_desc + off, kd + off, kIdescSq, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
      }
      __syncwarp();
      ++s_done;
      release_q();
      return true;
    };
    auto issue_dp = [&](int jj) -> bool {  // dP_jj = dO V_jj^T -> buffer g % 2, then V_jj is free
      const uint32_t g = kbase + jj;
      const int s = static_cast<int>(g % C::NV);
      if (!wait_all(v_full + s, (g / C::NV) & 1, abort, ctl, kSiteBwdMma)) return false;
      tc_fence_after();
      if (leader) {
        const SDesc vd = v_desc + s * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + kQColDP + (g & 1) * kT, do_desc + off, vd + off, kIdescSq,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(dp_full + (g & 1));
        mma_commit(v_empty + s);
      }
      __syncwarp();
      ++dp_done;
      release_q();
      return true;
    };
    // Order: S_0, dP_0, [S_0 read] S_1, dP_1, [dS_0] dQ_0, [S_1 read] S_2,
    // dP_2, [dS_1] dQ_1, ...: S_{j+1} overwrites S_j once both warpgroups
    // have read it, so the tensor core computes it while the softmax forms
    // dS_j; dP_{j+1} overwrites dS_{j-1} in the other buffer after dQ_{j-1}
    // has read it (same thread, in order).
    bool ok = true;
    int idx = 0;
    uint32_t q_items = 0;  // items with at least one key tile (one Q load each)
    for (int it = 0; ok; ++it) {
      if (!next_item(it, idx, kSiteBwdMma)) break;
      if (idx < 0) break;
      int bh, i;
      decode(idx, bh, i, n_kv);
      if (n_kv == 0) continue;  // the block mask hides every key from this query tile
      released = s_done = dp_done = 0;
      ok = wait_all(q_full, q_items & 1, abort, ctl, kSiteBwdMma) && issue_s(0) && issue_dp(0);
      ++q_items;
      for (int jj = 0; ok && jj < n_kv; ++jj) {
        const uint32_t g = kbase + jj;
        const int s = static_cast<int>(g % C::NK);
        if (jj + 1 < n_kv) {
          if (!wait_all(s_read, g & 1, abort, ctl, kSiteBwdMma) || !issue_s(jj + 1) ||
              !issue_dp(jj + 1)) {
            ok = false;
            break;
          }
        }
        // dQ += dS_jj K_jj: key k-step kk (16 keys) of dS at column
        // 64*(kk/4) + 8*(kk%4) of the dP buffer.  dS arrives in two parts
        // (k-steps with kk%4 < 2, then the rest); each part's MMAs go as soon
        // as it is in.
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          if (!wait_all(ds_full + 2 * (g & 1) + part, (g >> 1) & 1, abort, ctl, kSiteBwdMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
            const SDesc km = k_mn + s * C::TILE;
#pragma unroll
            for (int kh = 0; kh < 2; ++kh)
#pragma unroll
              for (int k2 = 0; k2 < 2; ++k2) {
                const int kk = 4 * kh + 2 * part + k2;
                mma_ts(tmem + kQColDQ,
                       tmem + kQColDP + (g & 1) * kT + (kk >> 2) * 64 + (kk & 3) * 8,
                       km + kk * 2048, kIdescDq, (jj > 0 || kk > 0) ? 1u : 0u);
              }
            if (part) mma_commit(k_empty + s);
          }
          __syncwarp();
        }
        if (!ok) break;
      }
      if (!ok) break;
      if (leader) mma_commit(dq_done);
      __syncwarp();
      kbase += static_cast<uint32_t>(n_kv);
    }
    __syncwarp();
  } else {
    // ------------------------- dS (warps 0-3: keys 0-63, 4-7: keys 64-127)
    const int h = warp >> 2;
    const int qr = threadIdx.x & 127;  // query row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // One arrival per warp once every lane's tcgen05 loads / stores are done.
    auto warp_arrive = [&](uint64_t* bar) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    uint32_t kbase = 0;    // key tiles of the previous items (dP buffer numbering)
    uint32_t q_items = 0;  // items with at least one key tile
    bool ok = true;
    int idx = 0;
    for (int it = 0; ok; ++it) {
      if (!next_item(it, idx, kSiteBwdSoftmax)) break;
      if (idx < 0) break;
      int bh, i, n_kv;
      decode(idx, bh, i, n_kv);
      const int q_idx = i * kT + qr;
      if (n_kv == 0) {
        // These queries see no key: dQ = 0 (block mask only).
        if (q_idx < N) {
          uint4* row = reinterpret_cast<uint4*>(dq + (static_cast<size_t>(bh) * N + q_idx) * D);
          for (int c = h; c < D / 8; c += 2) row[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      const float my_l2 = lse2[static_cast<size_t>(bh) * Np + q_idx];  // +inf past N
      const float my_d = dvec[static_cast<size_t>(bh) * Np + q_idx];
      TileCursor cur(n_t);
      for (int jj = 0; jj < n_kv; ++jj) {
        const int jt = BS ? cur.next(tiles) : jj;  // key tile of the step
        const uint32_t g = kbase + jj;
        const uint32_t col_dp = kQColDP + (g & 1) * kT + 64 * h;
        if (!wait_all(s_full, g & 1, abort, ctl, kSiteBwdSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[2][32];
        tmem_ld32(lane_base + kQColS + 64 * h, sv[0]);
        tmem_ld32(lane_base + kQColS + 64 * h + 32, sv[1]);
        tmem_wait_ld();
        warp_arrive(s_read);  // the S columns may take S_{j+1} now
        const int k0 = jt * kT + 64 * h;  // first key of this half
        // keys k visible to this query: k <= q_idx (causal) and k < N
        const int lim = min(N, CAUSAL ? q_idx + 1 : N) - k0;
        float p[64];
        if (__any_sync(0xffffffffu, lim < 64))
          dq_p_row<true>(sv, scale_log2, my_l2, lim, p);
        else
          dq_p_row<false>(sv, scale_log2, my_l2, lim, p);
        if (!wait_all(dp_full + (g & 1), (g >> 1) & 1, abort, ctl, kSiteBwdSoftmax)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t dpv[2][32];
        tmem_ld32(lane_base + col_dp, dpv[0]);
        tmem_ld32(lane_base + col_dp + 32, dpv[1]);
        tmem_wait_ld();
        // dS = P o (dP - D), formed as P dP - P D on column pairs, into the
        // first 32 of this half's dP columns (already read) in two parts of
        // 32 keys, each signalled as soon as it is stored.
        uint32_t dsk[32];
        const float2 nd2 = make_float2(-my_d, -my_d);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int c = 16 * part; c < 16 * part + 16; ++c) {
            const int c0 = 2 * c, c1 = 2 * c + 1;
            const float2 pp = make_float2(p[c0], p[c1]);
            const float2 r = __ffma2_rn(pp, make_float2(__uint_as_float(dpv[c0 >> 5][c0 & 31]),
                                                        __uint_as_float(dpv[c1 >> 5][c1 & 31])),
                                        __fmul2_rn(pp, nd2));
            dsk[c] = pack_bf16(r.x, r.y);
          }
          tmem_st16(lane_base + col_dp + 16 * part,
                    *reinterpret_cast<const uint32_t(*)[16]>(&dsk[16 * part]));
          tmem_wait_st();
          warp_arrive(ds_full + 2 * (g & 1) + part);
        }
      }
      if (!ok) break;
      // dq_done completes once per item; the next item's first dQ MMA
      // (accumulate off) comes after this warpgroup's next dS, so the loads
      // below are complete by then.
      if (!wait_all(dq_done, q_items & 1, abort, ctl, kSiteBwdEpilogue)) break;
      ++q_items;
      tc_fence_after();
      if constexpr (D == 128) {
        const int r0 = i * kT + (warp & 3) * 32;  // first query row of this warp
        const int nv = min(max(N - r0, 0), 32);
        store_rows_t128(lane_base + kQColDQ, scale, dq + (static_cast<size_t>(bh) * N + r0) * D, nv,
                        h, lane);
      } else {
        store_row_bf16<D>(lane_base + kQColDQ, scale,
                          dq + (static_cast<size_t>(bh) * N + q_idx) * D, q_idx < N, h, wide);
      }
      tc_fence_before();
      kbase += static_cast<uint32_t>(n_kv);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ launch

// Heads per group, from the bytes every item of a head re-reads (Q and dO for
// the dK/dV kernel, K and V for the dQ kernel: 4 N d each): a group's share
// stays within the L2 share (64 MB causal, 32 MB otherwise); causal groups
// are large so that the longest-first order ends on short items (small
// groups start their last group's long items at the end and leave SMs idle).
inline int heads_per_group(long long per_head_bytes, int BH, bool causal) {
  int g = static_cast<int>(l2_group_bytes(causal) / (per_head_bytes > 0 ? per_head_bytes : 1));
  return g < 1 ? 1 : (g > BH ? BH : g);
}

// Row statistics of the backward, one pass over O and dO: D = rowsum(dO o O)
// (fp32, columns in order) and LSE2 = LSE log2(e), in [BH, Np] vectors
// (Np = N rounded up to 128; rows past N get D = 0 and LSE2 = +inf, so a
// whole 128-row tile can be read without masks).  Half a warp per row, each
// lane one 16-byte piece of O and of dO (d / 8 lanes in use), so every load
// instruction moves whole rows.
template <int D>
__global__ void __launch_bounds__(256) row_stats_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dO,
                                                        const float* __restrict__ lse,
                                                        float* __restrict__ dvec,
                                                        float* __restrict__ lse2, int BH, int N,
                                                        int Np) {
  constexpr int kPieces = D / 8;  // 16-byte pieces per row
  static_assert(kPieces <= 16, "a row must fit half a warp");
  const int lane = threadIdx.x & 31, sub = lane & 15;
  const long long rows = static_cast<long long>(BH) * Np;
  const long long nwarps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  // Warp w handles rows 2w and 2w + 1 (one per half); all lanes take the
  // same trips, so the shuffles below always see the whole warp.
  for (long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       2 * w < rows; w += nwarps) {
    const long long r = 2 * w + (lane >> 4);
    const bool in = r < rows;
    const int bh = in ? static_cast<int>(r / Np) : 0;
    const int row = in ? static_cast<int>(r - static_cast<long long>(bh) * Np) : N;
    float acc = 0.f;
    if (row < N && sub < kPieces) {
      const size_t off = (static_cast<size_t>(bh) * N + row) * D + 8 * sub;
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + off));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(dO + off));
      acc = fmaf(bf16lo(a.x), bf16lo(b.x), acc);
      acc = fmaf(bf16hi(a.x), bf16hi(b.x), acc);
      acc = fmaf(bf16lo(a.y), bf16lo(b.y), acc);
      acc = fmaf(bf16hi(a.y), bf16hi(b.y), acc);
      acc = fmaf(bf16lo(a.z), bf16lo(b.z), acc);
      acc = fmaf(bf16hi(a.z), bf16hi(b.z), acc);
      acc = fmaf(bf16lo(a.w), bf16lo(b.w), acc);
      acc = fmaf(bf16hi(a.w), bf16hi(b.w), acc);
    }
#pragma unroll
    for (int m = 8; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (in && sub == 0) {
      dvec[r] = row < N ? acc : 0.f;
      lse2[r] = row < N ? lse[static_cast<size_t>(bh) * N + row] * 1.4426950408889634f
                        : INFINITY;
    }
  }
}

template <int D, bool CAUSAL, bool BS>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& tdo, const void* o, const void* dO, const float* lse,
                   float* dvec, float* lse2, void* dq, void* dk, void* dv, int BH, int N,
                   float scale, const BlockMaskArg& bm, const Launch& L) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, CAUSAL, BS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         KvCfg<D>::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_dq_kernel<D, CAUSAL, BS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, QCfg<D>::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_t = (N + kT - 1) / kT;
  const long long blocks = static_cast<long long>(BH) * n_t;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int group = heads_per_group(4LL * N * D, BH, CAUSAL);
  const float scale_log2 = scale * 1.4426950408889634f;
  WaitCtl ctl{L.status, L.limit_ns};
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long rows = static_cast<long long>(BH) * n_t * kT;
  const long long want = (rows + 15) / 16;  // 16 rows per 256-thread block
  const unsigned sblocks =
      static_cast<unsigned>(want < 8LL * sms ? (want < 1 ? 1 : want) : 8LL * sms);
  row_stats_kernel<D><<<sblocks, 256, 0, L.stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, dvec,
      lse2, BH, N, n_t * kT);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 32-byte row stores when every gradient tensor allows them (rows of
  // 128, 160 or 256 bytes keep a 32-byte aligned base aligned).
  const bool wide = ((reinterpret_cast<uintptr_t>(dq) | reinterpret_cast<uintptr_t>(dk) |
                      reinterpret_cast<uintptr_t>(dv)) & 31u) == 0;
  bwd_dq_kernel<D, CAUSAL, BS>
      <<<static_cast<unsigned>(blocks), kThreads, QCfg<D>::SMEM, L.stream>>>(
          tq, tk, tv, tdo, dvec, lse2, static_cast<__nv_bfloat16*>(dq), N, BH, group, scale,
          scale_log2, bm.mask, bm.mask_heads, bm.H, wide, ctl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D, CAUSAL, BS>
      <<<static_cast<unsigned>(blocks), kThreads, KvCfg<D>::SMEM, L.stream>>>(
          tq, tk, tv, tdo, dvec, lse2, static_cast<__nv_bfloat16*>(dk),
          static_cast<__nv_bfloat16*>(dv), N, BH, group, scale, scale_log2, bm.mask,
          bm.mask_heads, bm.H, wide, ctl);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, const void* o, const void* dO, const float* lse,
                     float* dvec, float* lse2, void* dq, void* dk, void* dv, int BH, int N,
                     float scale, int causal, const BlockMaskArg* bm, const Launch& L) {
  const BlockMaskArg none{nullptr, 1, 1};
  if (bm && bm->mask)
    return causal ? launch<D, true, true>(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv,
                                          BH, N, scale, *bm, L)
                  : launch<D, false, true>(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv,
                                           BH, N, scale, *bm, L);
  return causal ? launch<D, true, false>(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv, BH,
                                         N, scale, none, L)
                : launch<D, false, false>(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv,
                                          BH, N, scale, none, L);
}

}  // namespace bwd

cudaError_t launch_bwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const void* o, const void* dO,
                             const float* lse, float* dvec, float* lse2, void* dq, void* dk,
                             void* dv, int BH, int N, int d, float scale, int causal,
                             const BlockMaskArg* bm, const Launch& L) {
  switch (d) {
    case 64:
      return bwd::launch_d<64>(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv, BH, N, scale,
                               causal, bm, L);
    case 80:
      return bwd::launch_d<80>(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv, BH, N, scale,
                               causal, bm, L);
    case 128:
      return bwd::launch_d<128>(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv, BH, N,
                                scale, causal, bm, L);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace fa
