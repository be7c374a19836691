// fa_simt.cu -- CUDA-core kernels of the attention library:
//   * the fp32 forward and backward (fp32 FMA throughout, for accuracy
//     checks at small sizes; TF32 tensor cores cannot hold 1e-5),
//   * the fp32 backward's preprocess (D = rowsum(dO o O), padded to whole
//     128-row tiles; the bf16 backward computes D in its dQ kernel),
//   * the bounded-wait self test.
//
// The forward follows the blocked algorithm of the "FlashAttention-2" review
// page (core-algorithm answer, (2) forward pass): keys are visited in tiles
// staged in shared memory, each query row keeps a running max and running
// sum, and the output is normalised once at the end.  The backward follows
// the same page's (3) backward pass with the recomputation of P from the
// saved LSE ("[LLM] Flash Attention" blog, "Recomputation").
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace simt {

constexpr int kRows = 64;  // query (or key) rows per block, one thread each
constexpr int kKeys = 32;  // keys (or queries) staged per shared-memory tile
constexpr int kDMax = 128;

// ---------------------------------------------------------------- forward

__global__ void __launch_bounds__(kRows)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                   const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse,
                   int N, int d, float scale, int causal) {
  extern __shared__ float sh[];
  float* ks = sh;                  // [kKeys][d]
  float* vs = sh + kKeys * d;      // [kKeys][d]
  float* qs = sh + 2 * kKeys * d;  // [kRows][d + 1]
  const int bh = blockIdx.x;
  const int r0 = blockIdx.y * kRows;
  const int t = threadIdx.x;
  const int qi = r0 + t;
  const size_t base = static_cast<size_t>(bh) * N * d;
  for (int e = t; e < kRows * d; e += kRows) {
    const int rr = e / d, cc = e % d;
    qs[rr * (d + 1) + cc] = (r0 + rr < N) ? q[base + static_cast<size_t>(r0 + rr) * d + cc] : 0.f;
  }
  float acc[kDMax];
#pragma unroll
  for (int c = 0; c < kDMax; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int kend = causal ? min(N, r0 + kRows) : N;
  for (int k0 = 0; k0 < kend; k0 += kKeys) {
    __syncthreads();
    for (int e = t; e < kKeys * d; e += kRows) {
      const int rr = e / d, cc = e % d;
      const bool in = k0 + rr < N;
      ks[e] = in ? k[base + static_cast<size_t>(k0 + rr) * d + cc] : 0.f;
      vs[e] = in ? v[base + static_cast<size_t>(k0 + rr) * d + cc] : 0.f;
    }
    __syncthreads();
    const int nk = min(kKeys, N - k0);
    for (int jj = 0; jj < nk; ++jj) {
      const int kj = k0 + jj;
      if (causal && kj > qi) break;
      float dot = 0.f;
      for (int c = 0; c < d; ++c) dot = fmaf(qs[t * (d + 1) + c], ks[jj * d + c], dot);
      const float s = dot * scale;
      if (s > m) {
        const float corr = expf(m - s);  // 0 when m = -inf
        l *= corr;
#pragma unroll
        for (int c = 0; c < kDMax; ++c) acc[c] *= corr;
        m = s;
      }
      const float p = expf(s - m);
      l += p;
#pragma unroll
      for (int c = 0; c < kDMax; ++c)
        if (c < d) acc[c] = fmaf(p, vs[jj * d + c], acc[c]);
    }
  }
  if (qi < N) {
    const float inv = 1.f / l;
#pragma unroll
    for (int c = 0; c < kDMax; ++c)
      if (c < d) o[base + static_cast<size_t>(qi) * d + c] = acc[c] * inv;
    lse[static_cast<size_t>(bh) * N + qi] = m + logf(l);
  }
}

// --------------------------------------------------------------- backward
// Two passes without atomics: dK/dV with one thread per key row looping over
// queries, dQ with one thread per query row looping over keys.

__global__ void __launch_bounds__(kRows)
    bwd_dkdv_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                        const float* __restrict__ v, const float* __restrict__ dO,
                        const float* __restrict__ lse, const float* __restrict__ dvec,
                        float* __restrict__ dk, float* __restrict__ dv, int N, int Np, int d,
                        float scale, int causal) {
  extern __shared__ float sh[];
  float* qs = sh;                  // [kKeys][d]
  float* ds_ = sh + kKeys * d;     // dO tile [kKeys][d]
  float* ks = sh + 2 * kKeys * d;  // [kRows][d+1]
  float* vsh = ks + kRows * (d + 1);
  __shared__ float lse_s[kKeys], d_s[kKeys];
  const int bh = blockIdx.x;
  const int r0 = blockIdx.y * kRows;
  const int t = threadIdx.x;
  const int kj = r0 + t;
  const size_t base = static_cast<size_t>(bh) * N * d;
  for (int e = t; e < kRows * d; e += kRows) {
    const int rr = e / d, cc = e % d;
    const bool in = r0 + rr < N;
    ks[rr * (d + 1) + cc] = in ? k[base + static_cast<size_t>(r0 + rr) * d + cc] : 0.f;
    vsh[rr * (d + 1) + cc] = in ? v[base + static_cast<size_t>(r0 + rr) * d + cc] : 0.f;
  }
  float adk[kDMax], adv[kDMax];
#pragma unroll
  for (int c = 0; c < kDMax; ++c) adk[c] = adv[c] = 0.f;
  const int q_start = causal ? r0 : 0;
  for (int i0 = q_start; i0 < N; i0 += kKeys) {
    __syncthreads();
    for (int e = t; e < kKeys * d; e += kRows) {
      const int rr = e / d, cc = e % d;
      const bool in = i0 + rr < N;
      qs[e] = in ? q[base + static_cast<size_t>(i0 + rr) * d + cc] : 0.f;
      ds_[e] = in ? dO[base + static_cast<size_t>(i0 + rr) * d + cc] : 0.f;
    }
    for (int e = t; e < kKeys; e += kRows) {
      const bool in = i0 + e < N;
      lse_s[e] = in ? lse[static_cast<size_t>(bh) * N + i0 + e] : 0.f;
      d_s[e] = in ? dvec[static_cast<size_t>(bh) * Np + i0 + e] : 0.f;
    }
    __syncthreads();
    const int nq = min(kKeys, N - i0);
    for (int ii = 0; ii < nq; ++ii) {
      const int qi = i0 + ii;
      if (causal && kj > qi) continue;
      float sdot = 0.f, dpdot = 0.f;
      for (int c = 0; c < d; ++c) {
        sdot = fmaf(qs[ii * d + c], ks[t * (d + 1) + c], sdot);
        dpdot = fmaf(ds_[ii * d + c], vsh[t * (d + 1) + c], dpdot);
      }
      const float p = expf(sdot * scale - lse_s[ii]);
      const float dsv = p * (dpdot - d_s[ii]);
#pragma unroll
      for (int c = 0; c < kDMax; ++c) {
        if (c < d) {
          adv[c] = fmaf(p, ds_[ii * d + c], adv[c]);
          adk[c] = fmaf(dsv, qs[ii * d + c], adk[c]);
        }
      }
    }
  }
  if (kj < N) {
#pragma unroll
    for (int c = 0; c < kDMax; ++c) {
      if (c < d) {
        dk[base + static_cast<size_t>(kj) * d + c] = adk[c] * scale;
        dv[base + static_cast<size_t>(kj) * d + c] = adv[c];
      }
    }
  }
}

__global__ void __launch_bounds__(kRows)
    bwd_dq_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                      const float* __restrict__ v, const float* __restrict__ dO,
                      const float* __restrict__ lse, const float* __restrict__ dvec,
                      float* __restrict__ dq, int N, int Np, int d, float scale, int causal) {
  extern __shared__ float sh[];
  float* ks = sh;                   // [kKeys][d]
  float* vsh = sh + kKeys * d;      // [kKeys][d]
  float* qs = sh + 2 * kKeys * d;   // [kRows][d+1]
  float* dos = qs + kRows * (d + 1);
  const int bh = blockIdx.x;
  const int r0 = blockIdx.y * kRows;
  const int t = threadIdx.x;
  const int qi = r0 + t;
  const size_t base = static_cast<size_t>(bh) * N * d;
  for (int e = t; e < kRows * d; e += kRows) {
    const int rr = e / d, cc = e % d;
    const bool in = r0 + rr < N;
    qs[rr * (d + 1) + cc] = in ? q[base + static_cast<size_t>(r0 + rr) * d + cc] : 0.f;
    dos[rr * (d + 1) + cc] = in ? dO[base + static_cast<size_t>(r0 + rr) * d + cc] : 0.f;
  }
  const float my_lse = qi < N ? lse[static_cast<size_t>(bh) * N + qi] : 0.f;
  const float my_d = qi < N ? dvec[static_cast<size_t>(bh) * Np + qi] : 0.f;
  float adq[kDMax];
#pragma unroll
  for (int c = 0; c < kDMax; ++c) adq[c] = 0.f;
  const int kend = causal ? min(N, r0 + kRows) : N;
  for (int k0 = 0; k0 < kend; k0 += kKeys) {
    __syncthreads();
    for (int e = t; e < kKeys * d; e += kRows) {
      const int rr = e / d, cc = e % d;
      const bool in = k0 + rr < N;
      ks[e] = in ? k[base + static_cast<size_t>(k0 + rr) * d + cc] : 0.f;
      vsh[e] = in ? v[base + static_cast<size_t>(k0 + rr) * d + cc] : 0.f;
    }
    __syncthreads();
    const int nk = min(kKeys, N - k0);
    for (int jj = 0; jj < nk; ++jj) {
      const int kj = k0 + jj;
      if (causal && kj > qi) break;
      float sdot = 0.f, dpdot = 0.f;
      for (int c = 0; c < d; ++c) {
        sdot = fmaf(qs[t * (d + 1) + c], ks[jj * d + c], sdot);
        dpdot = fmaf(dos[t * (d + 1) + c], vsh[jj * d + c], dpdot);
      }
      const float p = expf(sdot * scale - my_lse);
      const float dsv = p * (dpdot - my_d);
#pragma unroll
      for (int c = 0; c < kDMax; ++c)
        if (c < d) adq[c] = fmaf(dsv, ks[jj * d + c], adq[c]);
    }
  }
  if (qi < N) {
#pragma unroll
    for (int c = 0; c < kDMax; ++c)
      if (c < d) dq[base + static_cast<size_t>(qi) * d + c] = adq[c] * scale;
  }
}

// ------------------------------------------------------------- preprocess
// One warp per (head, padded row).  Rows N..Np-1 of the row vectors get
// D = 0 and lse2 = +inf, so a kernel reading a whole 128-row tile computes
// P = 2^(s - inf) = 0 there.
template <typename T>
__device__ __forceinline__ float ld_as_float(const T* p, size_t i);
template <>
__device__ __forceinline__ float ld_as_float<float>(const float* p, size_t i) {
  return p[i];
}
template <>
__device__ __forceinline__ float ld_as_float<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

template <typename T>
__global__ void bwd_preprocess_kernel(const T* __restrict__ o, const T* __restrict__ dO,
                                      const float* __restrict__ lse, float* __restrict__ dvec,
                                      float* __restrict__ lse2, int BH, int N, int Np, int d) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= BH * Np) return;
  const int bh = gw / Np;
  const int row = gw % Np;
  float acc = 0.f;
  if (row < N) {
    const size_t base = (static_cast<size_t>(bh) * N + row) * d;
    for (int c = lane; c < d; c += 32) {
      acc = fmaf(ld_as_float(dO, base + c), ld_as_float(o, base + c), acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const size_t vi = static_cast<size_t>(bh) * Np + row;
    dvec[vi] = row < N ? acc : 0.f;
    if (lse2)
      lse2[vi] = row < N ? lse[static_cast<size_t>(bh) * N + row] * 1.4426950408889634f : INFINITY;
  }
}

// A barrier nothing ever arrives on: the bounded wait must give up, record
// its site and return.
__global__ void selftest_wait_kernel(WaitCtl ctl) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort, ctl, kSiteSelfTest);
  __syncthreads();
}

// Merge of split-KV partials, one warp per output row: LSE = m + ln S,
// S = sum_s e^(LSE_s - m), m = max_s LSE_s, and O = sum_s e^(LSE_s - m) O_s / S
// ("FlashAttention-2" review: the online-softmax merge of running max and
// sum, applied across the key splits).  Rows whose splits all saw no key
// (every LSE_s = -inf) get O = 0 and LSE = -inf.
__global__ void splitkv_combine_kernel(const float* __restrict__ part_o,
                                       const float* __restrict__ part_lse,
                                       __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                       int n_split, int rows, int d) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int s = 0; s < n_split; ++s)
    m = fmaxf(m, part_lse[static_cast<size_t>(s) * rows + row]);
  __nv_bfloat16* orow = o + static_cast<size_t>(row) * d;
  if (m == -INFINITY) {
    for (int c = lane; c < d; c += 32) orow[c] = __float2bfloat16(0.f);
    if (lane == 0) lse[row] = -INFINITY;
    return;
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // columns lane, lane + 32, lane + 64, lane + 96
  float tot = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float ls = part_lse[static_cast<size_t>(s) * rows + row];
    if (ls == -INFINITY) continue;
    const float w = expf(ls - m);
    tot += w;
    const float* prow = part_o + (static_cast<size_t>(s) * rows + row) * d;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (lane + 32 * e < d) acc[e] += w * prow[lane + 32 * e];
  }
  const float inv = 1.f / tot;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (lane + 32 * e < d) orow[lane + 32 * e] = __float2bfloat16(acc[e] * inv);
  if (lane == 0) lse[row] = m + logf(tot);
}

}  // namespace simt

static int blocks_for(size_t work, int per_block) {
  size_t b = (work + per_block - 1) / per_block;
  return static_cast<int>(b > 0x7fffffff ? 0x7fffffff : b);
}

cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int BH, int N, int d, float scale, int causal, const Launch& L) {
  const size_t smem = (2 * simt::kKeys * d + simt::kRows * (d + 1)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(simt::fwd_f32_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(BH, (N + simt::kRows - 1) / simt::kRows);
  simt::fwd_f32_kernel<<<grid, simt::kRows, smem, L.stream>>>(q, k, v, o, lse, N, d, scale,
                                                              causal);
  return cudaGetLastError();
}

cudaError_t launch_bwd_f32(const float* q, const float* k, const float* v, const float* dO,
                           const float* lse, const float* dvec, float* dq, float* dk, float* dv,
                           int BH, int N, int d, float scale, int causal, const Launch& L) {
  const size_t smem = (2 * simt::kKeys * d + 2 * simt::kRows * (d + 1)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(simt::bwd_dkdv_f32_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(simt::bwd_dq_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(BH, (N + simt::kRows - 1) / simt::kRows);
  const int Np = round_up(N, kTileRows);  // row stride of dvec
  simt::bwd_dkdv_f32_kernel<<<grid, simt::kRows, smem, L.stream>>>(q, k, v, dO, lse, dvec, dk,
                                                                   dv, N, Np, d, scale, causal);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  simt::bwd_dq_f32_kernel<<<grid, simt::kRows, smem, L.stream>>>(q, k, v, dO, lse, dvec, dq, N,
                                                                 Np, d, scale, causal);
  return cudaGetLastError();
}

cudaError_t launch_bwd_preprocess(const void* o, const void* dO, const float* lse, float* dvec,
                                  float* lse2, int BH, int N, int d, int is_bf16,
                                  const Launch& L) {
  const int Np = round_up(N, kTileRows);
  const size_t warps = static_cast<size_t>(BH) * Np;
  const int threads = 256;
  const int blocks = blocks_for(warps * 32, threads);
  if (is_bf16)
    simt::bwd_preprocess_kernel<__nv_bfloat16><<<blocks, threads, 0, L.stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, dvec,
        lse2, BH, N, Np, d);
  else
    simt::bwd_preprocess_kernel<float><<<blocks, threads, 0, L.stream>>>(
        static_cast<const float*>(o), static_cast<const float*>(dO), lse, dvec, lse2, BH, N, Np,
        d);
  return cudaGetLastError();
}

cudaError_t launch_splitkv_combine(const float* part_o, const float* part_lse, void* o,
                                   float* lse, int n_split, int rows, int d, const Launch& L) {
  if (d > 128) return cudaErrorInvalidValue;
  const int threads = 256;
  const int blocks = blocks_for(static_cast<size_t>(rows) * 32, threads);
  simt::splitkv_combine_kernel<<<blocks, threads, 0, L.stream>>>(
      part_o, part_lse, static_cast<__nv_bfloat16*>(o), lse, n_split, rows, d);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(const Launch& L) {
  WaitCtl ctl{L.status, L.limit_ns};
  simt::selftest_wait_kernel<<<1, 32, 0, L.stream>>>(ctl);
  return cudaGetLastError();
}

}  // namespace fa
