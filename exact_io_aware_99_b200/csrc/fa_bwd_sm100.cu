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
// B200 design: one CTA per (head, 128-key tile K_j/V_j), looping over the
// query tiles Q_i that see it (all of them, or i >= j when causal), so the
// work is parallel over batch, head and sequence as FA2 prescribes
// ("FlashAttention-2" review, results answer, parallelism over sequence
// length).  10 warps:
//   warp 8      TMA producer: K_j, V_j once; Q_i and dO_i into a 2-stage ring.
//   warp 9      TMEM allocator and single-thread MMA issuer, per Q tile:
//                 S^T  = K_j Q_i^T   -> TMEM cols [0,128)    (SS)
//                 dP^T = V_j dO_i^T  -> TMEM cols [128,256)  (SS)
//                 dV  += P^T dO_i    -> TMEM cols [256,256+d) (TS: P^T from TMEM)
//                 dK  += dS^T Q_i    -> TMEM cols [384,384+d) (SS, dS^T from smem)
//                 dQ_i = dS K_j      -> TMEM cols [128,128+d) (SS, dS read MN-major)
//   warps 0-3   one thread per key row: P^T = 2^(S^T c - LSE2) written back to
//               TMEM as bf16 over S^T; dS^T = P^T o (dP^T - D) written to
//               shared memory in the 128-byte-swizzled layout the MMAs read.
//   warps 4-7   one thread per query row: read dQ_i from TMEM, scale, stage
//               it (fp32, 128-byte swizzled) in the dS buffer once the dK/dQ
//               MMAs are done with it, and add it to the fp32 dQ accumulator
//               with TMA tensor reductions (whole 128-byte lines); then the dK
//               epilogue (warps 0-3 do dV).
// TMEM holds 512 columns, so dQ_i reuses the dP^T columns: S^T_{i+1} is
// issued right behind dQ_i and overlaps the dQ readout; dP^T_{i+1} waits for
// the readout.  CTAs run group-major (a few heads at a time, so their K, V,
// Q, dO and dQ accumulator stay in L2), longest-first inside a group.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int kBM = 128;  // keys per CTA (TMEM lanes of S^T, dP^T, dK, dV)
constexpr int kBN = 128;  // queries per inner tile
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

template <int D>
struct Cfg {
  static constexpr int NB = (D + 63) / 64;
  static constexpr int BLK = 64 * 128 * 2;  // one 128-row x 64-col bf16 swizzle block
  static constexpr int TILE = NB * BLK;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + TILE;
  static constexpr int Q_OFF = V_OFF + TILE;      // [2] stages
  static constexpr int DO_OFF = Q_OFF + 2 * TILE; // [2] stages
  static constexpr int DS_OFF = DO_OFF + 2 * TILE;
  static constexpr int DS_BYTES = 2 * BLK;        // 128 keys x 128 queries bf16
  static constexpr int BAR_OFF = DS_OFF + DS_BYTES;
  static constexpr int NBAR = 16;
  static constexpr int NSUB = (D + 31) / 32;      // 32-column fp32 dQ sub-tiles
  static_assert(DS_BYTES >= 4 * 2 * 4096, "dQ staging: 4 warps x 2 sub-tiles of 32x32 fp32");
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;
  static constexpr int KSTEPS = D / 16;
  static_assert(D % 16 == 0 && D <= 128, "head dim must be a multiple of 16, <= 128");
  static_assert(SMEM <= 232448, "shared memory budget");
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

// Store 8 consecutive bf16 (one 16-byte chunk) of row `row`, chunk `chunk`
// (0..15 over 128 columns) of a 128-row tile in the 128-byte-swizzled layout:
// 64-column blocks of 128 x 128 B, chunk index XOR (row mod 8).
__device__ __forceinline__ void st_sw128(uint8_t* tile, int row, int chunk, uint4 val) {
  const int blk = chunk >> 3;
  const int c = (chunk & 7) ^ (row & 7);
  *reinterpret_cast<uint4*>(tile + blk * (64 * 128 * 2) + row * 128 + c * 16) = val;
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const float* __restrict__ dvec,
               const float* __restrict__ lse2, __nv_bfloat16* __restrict__ dk,
               __nv_bfloat16* __restrict__ dv, int N, int BH, int group, float scale,
               float scale_log2, WaitCtl ctl) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;     // [2]
  uint64_t* do_full = bars + 3;    // [2]
  uint64_t* qdo_empty = bars + 5;  // [2]
  uint64_t* s_full = bars + 7;
  uint64_t* dp_full = bars + 8;
  uint64_t* p_full = bars + 9;
  uint64_t* ds_full = bars + 10;
  uint64_t* dq_full = bars + 11;
  uint64_t* dq_empty = bars + 12;  // dQ read out of TMEM (dP^T columns free)
  uint64_t* ds_free = bars + 13;   // dQ staging done with the dS buffer
  uint64_t* kv_done = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  const int warp = warp_id();
  const int lane = lane_id();
  const int n_q = (N + kBN - 1) / kBN;
  // Group-major order: `group` heads at a time, and inside a group key tile
  // j ascending (j = 0 has the most work when causal), head fastest.
  int bh, j;
  {
    const int per_group = group * n_q;
    const int g = static_cast<int>(blockIdx.x) / per_group;
    const int r = static_cast<int>(blockIdx.x) - g * per_group;
    const int gh = min(group, BH - g * group);
    j = r / gh;
    bh = g * group + (r - j * gh);
  }
  const int Np = n_q * kBN;
  const int i_start = CAUSAL ? j : 0;
  const int n_iter = n_q - i_start;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(do_full + s, 1);
      mbar_init(qdo_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, kBM);
    mbar_init(ds_full, kBM);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, kBN);
    mbar_init(ds_free, 4);
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

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      int last[2] = {-1, -1};
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
#pragma unroll
      for (int b = 0; b < C::NB; ++b) {
        tma_load_3d(&tm_k, kv_full, smem + C::K_OFF + b * C::BLK, b * 64, j * kBM, bh);
        tma_load_3d(&tm_v, kv_full, smem + C::V_OFF + b * C::BLK, b * 64, j * kBM, bh);
      }
      for (int it = 0; it < n_iter; ++it) {
        const int st = it & 1;
        const uint32_t u = static_cast<uint32_t>(it >> 1);
        if (it >= 2 && !mbar_wait(qdo_empty + st, (u - 1) & 1, abort, ctl, kSiteBwdProducer))
          break;
        const int y = (i_start + it) * kBN;
        mbar_arrive_expect_tx(q_full + st, C::TILE);
#pragma unroll
        for (int b = 0; b < C::NB; ++b)
          tma_load_3d(&tm_q, q_full + st, smem + C::Q_OFF + st * C::TILE + b * C::BLK, b * 64, y,
                      bh);
        mbar_arrive_expect_tx(do_full + st, C::TILE);
#pragma unroll
        for (int b = 0; b < C::NB; ++b)
          tma_load_3d(&tm_do, do_full + st, smem + C::DO_OFF + st * C::TILE + b * C::BLK, b * 64,
                      y, bh);
        last[st] = static_cast<int>(u);
      }
      if (*abort) {
        drain_wait(kv_full, 0, ctl);
        for (int s = 0; s < 2; ++s)
          if (last[s] >= 0) {
            drain_wait(q_full + s, last[s] & 1, ctl);
            drain_wait(do_full + s, last[s] & 1, ctl);
          }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescSq = idesc_bf16(kBM, kBN, 0, 0);  // S^T, dP^T
      constexpr uint32_t kIdescAcc = idesc_bf16(kBM, D, 0, 1);   // dV, dK (B MN-major)
      constexpr uint32_t kIdescDq = idesc_bf16(kBN, D, 1, 1);    // dQ (A and B MN-major)
      const uint32_t k_addr = sbase + C::K_OFF;
      const uint32_t v_addr = sbase + C::V_OFF;
      const uint32_t ds_addr = sbase + C::DS_OFF;
      auto issue_s = [&](int it) -> bool {  // S^T = K_j Q_i^T -> cols [0,128)
        const int st = it & 1;
        if (!mbar_wait(q_full + st, static_cast<uint32_t>(it >> 1) & 1, abort, ctl, kSiteBwdMma))
          return false;
        tc_fence_after();
        const uint32_t q_addr = sbase + C::Q_OFF + st * C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + kColS, sdesc_sw128(k_addr + off, 16, 1024),
                 sdesc_sw128(q_addr + off, 16, 1024), kIdescSq, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, abort, ctl, kSiteBwdMma) && issue_s(0);
      for (int it = 0; ok && it < n_iter; ++it) {
        const int st = it & 1;
        const uint32_t ph = static_cast<uint32_t>(it >> 1) & 1;
        const uint32_t q_addr = sbase + C::Q_OFF + st * C::TILE;
        const uint32_t do_addr = sbase + C::DO_OFF + st * C::TILE;
        // dP^T = V_j dO_i^T -> cols [128,256), once dQ_{i-1} has been read out.
        if (!mbar_wait(do_full + st, ph, abort, ctl, kSiteBwdMma)) break;
        if (it > 0 && !mbar_wait(dq_empty, (it - 1) & 1, abort, ctl, kSiteBwdMma)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + kColDP, sdesc_sw128(v_addr + off, 16, 1024),
                 sdesc_sw128(do_addr + off, 16, 1024), kIdescSq, kk > 0 ? 1u : 0u);
        }
        mma_commit(dp_full);
        // dV += P^T dO_i, P^T read from TMEM.
        if (!mbar_wait(p_full, it & 1, abort, ctl, kSiteBwdMma)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(tmem + kColDV, tmem + kColS + kk * 8,
                 sdesc_sw128(do_addr + kk * 2048, C::BLK, 1024), kIdescAcc,
                 (it > 0 || kk > 0) ? 1u : 0u);
        // dK += dS^T Q_i and dQ_i = dS K_j (into the dP^T columns).
        if (!mbar_wait(ds_full, it & 1, abort, ctl, kSiteBwdMma)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(tmem + kColDK, sdesc_sw128(ds_addr + off, 16, 1024),
                 sdesc_sw128(q_addr + kk * 2048, C::BLK, 1024), kIdescAcc,
                 (it > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk)
          mma_ss(tmem + kColDP, sdesc_sw128(ds_addr + kk * 2048, C::BLK, 1024),
                 sdesc_sw128(k_addr + kk * 2048, C::BLK, 1024), kIdescDq, kk > 0 ? 1u : 0u);
        mma_commit(dq_full);
        mma_commit(qdo_empty + st);
        // S^T of the next query tile overlaps the dQ readout.
        if (it + 1 < n_iter) ok = issue_s(it + 1);
      }
      mma_commit(kv_done);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------- P^T and dS^T (warps 0..3)
    const int kr = threadIdx.x;  // key row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int k_idx = j * kBM + kr;
    const bool key_ok = k_idx < N;
    uint8_t* ds_tile = smem + C::DS_OFF;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int i = i_start + it;
      const float* l2 = lse2 + static_cast<size_t>(bh) * Np + i * kBN;
      const float* dd = dvec + static_cast<size_t>(bh) * Np + i * kBN;
      const bool diag = CAUSAL && (i == j);
      if (!wait_all(s_full, it & 1, abort, ctl, kSiteBwdSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t sv[32];
        tmem_ld32(lane_base + kColS + c * 32, sv);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 lv = __ldg(reinterpret_cast<const float4*>(l2 + c * 32 + e));
          float p[4];
          p[0] = ex2(fmaf(__uint_as_float(sv[e + 0]), scale_log2, -lv.x));
          p[1] = ex2(fmaf(__uint_as_float(sv[e + 1]), scale_log2, -lv.y));
          p[2] = ex2(fmaf(__uint_as_float(sv[e + 2]), scale_log2, -lv.z));
          p[3] = ex2(fmaf(__uint_as_float(sv[e + 3]), scale_log2, -lv.w));
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int qcol = c * 32 + e + t;
            if (!key_ok || (diag && qcol < kr)) p[t] = 0.f;
          }
          pk[e / 2] = pack_bf16(p[0], p[1]);
          pk[e / 2 + 1] = pack_bf16(p[2], p[3]);
        }
        // P^T columns [16c, 16c+16) lie in S^T columns already read.
        tmem_st16(lane_base + kColS + c * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);

      // dS^T needs the dS buffer back (dK/dQ MMAs and the dQ staging of
      // iteration it-1 are done with it) and dP^T of this iteration.
      if (it > 0 && !wait_all(ds_free, (it - 1) & 1, abort, ctl, kSiteBwdSoftmax)) {
        ok = false;
        break;
      }
      if (!wait_all(dp_full, it & 1, abort, ctl, kSiteBwdSoftmax)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t dpv[32], pk[16];
        tmem_ld32(lane_base + kColDP + c * 32, dpv);
        tmem_ld16(lane_base + kColS + c * 16, pk);
        tmem_wait_ld();
        uint32_t dsk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 dv4 = __ldg(reinterpret_cast<const float4*>(dd + c * 32 + e));
          const float d0 = bf16lo(pk[e / 2]) * (__uint_as_float(dpv[e + 0]) - dv4.x);
          const float d1 = bf16hi(pk[e / 2]) * (__uint_as_float(dpv[e + 1]) - dv4.y);
          const float d2 = bf16lo(pk[e / 2 + 1]) * (__uint_as_float(dpv[e + 2]) - dv4.z);
          const float d3 = bf16hi(pk[e / 2 + 1]) * (__uint_as_float(dpv[e + 3]) - dv4.w);
          dsk[e / 2] = pack_bf16(d0, d1);
          dsk[e / 2 + 1] = pack_bf16(d2, d3);
        }
#pragma unroll
        for (int h = 0; h < 4; ++h)
          st_sw128(ds_tile, kr, c * 4 + h,
                   make_uint4(dsk[4 * h], dsk[4 * h + 1], dsk[4 * h + 2], dsk[4 * h + 3]));
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // dV epilogue
    if (ok && wait_all(kv_done, 0, abort, ctl, kSiteBwdEpilogue)) {
      tc_fence_after();
      uint4* row = reinterpret_cast<uint4*>(dv + (static_cast<size_t>(bh) * N + k_idx) * D);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t v16[16];
        tmem_ld16(lane_base + kColDV + c * 16, v16);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          pk[e] = pack_bf16(__uint_as_float(v16[2 * e]), __uint_as_float(v16[2 * e + 1]));
        if (key_ok) {
          row[2 * c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          row[2 * c + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  } else {
    // --------------------------------------------- dQ readout (warps 4..7)
    const int wq = warp - 4;           // TMEM lane quarter: query rows 32*wq..
    const int qr = threadIdx.x - 128;  // query row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    // Per-warp staging: two 32 x 32 fp32 sub-tiles (4 KB each, 128-byte
    // swizzled) inside the dS buffer.
    uint8_t* stage = smem + C::DS_OFF + wq * 8192;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int q0 = (i_start + it) * kBN;
      if (!wait_all(dq_full, it & 1, abort, ctl, kSiteBwdDq)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int pass = 0; pass < (C::NSUB + 1) / 2; ++pass) {
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int sub = 2 * pass + sl;
          if (sub < C::NSUB) {
            uint32_t v[32];
            tmem_ld32(lane_base + kColDP + sub * 32, v);
            tmem_wait_ld();
            uint8_t* rowp = stage + sl * 4096 + lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 f = make_float4(__uint_as_float(v[4 * c]) * scale,
                                           __uint_as_float(v[4 * c + 1]) * scale,
                                           __uint_as_float(v[4 * c + 2]) * scale,
                                           __uint_as_float(v[4 * c + 3]) * scale);
              *reinterpret_cast<float4*>(rowp + ((c ^ (lane & 7)) * 16)) = f;
            }
          }
        }
        if (2 * pass + 2 >= C::NSUB) {
          // Last TMEM read of dQ_i: release the dP^T columns.
          tc_fence_before();
          mbar_arrive(dq_empty);
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          const int y = q0 + wq * 32;
          if (y < N) {
#pragma unroll
            for (int sl = 0; sl < 2; ++sl)
              if (2 * pass + sl < C::NSUB)
                tma_reduce_add_3d(&tm_dq, stage + sl * 4096, (2 * pass + sl) * 32, y, bh);
          }
          bulk_commit();
          bulk_wait_read_all();
        }
        __syncwarp();
      }
      if (lane == 0) mbar_arrive(ds_free);
      (void)qr;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    // dK epilogue
    if (ok && wait_all(kv_done, 0, abort, ctl, kSiteBwdEpilogue)) {
      tc_fence_after();
      const int k_idx = j * kBM + qr;
      uint4* row = reinterpret_cast<uint4*>(dk + (static_cast<size_t>(bh) * N + k_idx) * D);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t v16[16];
        tmem_ld16(lane_base + kColDK + c * 16, v16);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          pk[e] = pack_bf16(__uint_as_float(v16[2 * e]) * scale,
                            __uint_as_float(v16[2 * e + 1]) * scale);
        if (k_idx < N) {
          row[2 * c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          row[2 * c + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
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
                   const CUtensorMap& tdo, const CUtensorMap& tdq, const float* dvec,
                   const float* lse2, void* dk, void* dv, int BH, int N, float scale,
                   const Launch& L) {
  using C = Cfg<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(bwd_kernel<D, CAUSAL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_kv = (N + kBM - 1) / kBM;
  // Heads per group: keep a group's K, V, Q, dO (bf16) and dQ accumulator
  // (fp32), 12 N d bytes per head, within ~48 MB of the 126 MB L2.
  const long long per_head = 12LL * N * D;
  int group = static_cast<int>((48LL << 20) / (per_head > 0 ? per_head : 1));
  group = group < 1 ? 1 : (group > BH ? BH : group);
  const long long blocks = static_cast<long long>(BH) * n_kv;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  WaitCtl ctl{L.status, L.limit_ns};
  bwd_kernel<D, CAUSAL><<<static_cast<unsigned>(blocks), kThreads, C::SMEM, L.stream>>>(
      tq, tk, tv, tdo, tdq, dvec, lse2, static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv), N, BH, group, scale, scale * 1.4426950408889634f, ctl);
  return cudaGetLastError();
}

}  // namespace bwd

cudaError_t launch_bwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const CUtensorMap& tdq, const float* dvec,
                             const float* lse2, void* dk, void* dv, int BH, int N, int d,
                             float scale, int causal, const Launch& L) {
#define FA_BWD_CASE(DD)                                                                     \
  case DD:                                                                                  \
    return causal ? bwd::launch<DD, true>(tq, tk, tv, tdo, tdq, dvec, lse2, dk, dv, BH, N,  \
                                          scale, L)                                         \
                  : bwd::launch<DD, false>(tq, tk, tv, tdo, tdq, dvec, lse2, dk, dv, BH, N, \
                                           scale, L);
  switch (d) {
    FA_BWD_CASE(64)
    FA_BWD_CASE(80)
    FA_BWD_CASE(128)
    default:
      return cudaErrorInvalidValue;
  }
#undef FA_BWD_CASE
}

}  // namespace fa
