// fa_internal.h -- launch interface between the C ABI (fa_api.cu) and the
// kernel translation units.  Not installed; not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

struct Launch {
  cudaStream_t stream;
  int* status;                  // device status word
  unsigned long long limit_ns;  // bounded-wait time limit
};

// Wait-site codes recorded in the status word when a bounded wait runs out.
enum WaitSite : int {
  kSiteFwdProducer = 0x101,
  kSiteFwdMma = 0x102,
  kSiteFwdSoftmax = 0x103,
  kSiteFwdEpilogue = 0x104,
  kSiteFwdDrain = 0x105,
  kSiteBwdProducer = 0x201,
  kSiteBwdMma = 0x202,
  kSiteBwdSoftmax = 0x203,
  kSiteBwdDq = 0x204,
  kSiteBwdEpilogue = 0x205,
  kSiteBwdDrain = 0x206,
  kSiteBwdSmem = 0x207,  // dynamic shared memory base needed more alignment slack than left
  kSiteSelfTest = 0x7e57,
};

// Rows of a head are padded to a multiple of this in the backward's row
// vectors (D and the base-2 LSE), and it is the tile height of every kernel.
constexpr int kTileRows = 128;

inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

// L2 share (MB) for the operands a group of heads keeps re-reading; it sets
// how many heads the kernels work on at a time (group-major work order).
// Causal launches take larger groups: their work items differ in length and
// a longest-first order only balances the SMs when it spans many heads.
// Non-causal items are all equal, so smaller groups (fewer L2 misses) win.
#ifndef FA_L2_GROUP_MB
#define FA_L2_GROUP_MB 64
#endif
#ifndef FA_L2_GROUP_MB_NONCAUSAL
#define FA_L2_GROUP_MB_NONCAUSAL 32
#endif
inline long long l2_group_bytes(int causal) {
  return static_cast<long long>(causal ? FA_L2_GROUP_MB : FA_L2_GROUP_MB_NONCAUSAL) << 20;
}

// Block mask of block-sparse attention: mask[(hm * n_t + i) * n_t + j] != 0
// lets query tile i (128 rows) see key tile j, n_t = ceil(N / 128); hm = 0
// when mask_heads == 1 (one mask for every head), else hm = (b * H + h) % H.
struct BlockMaskArg {
  const uint8_t* mask;  // device pointer; nullptr = dense
  int mask_heads;       // 1 or H
  int H;                // heads per batch entry
};

// Split-KV forward (decode): N_q queries against N_k keys, the key tiles of
// every (head, query tile pair) split into n_split ranges of kt_per tiles;
// each range writes a partial O (fp32, normalised over its keys) and LSE to
// part_o [n_split, BH, N_q, d] / part_lse [n_split, BH, N_q], merged by
// launch_splitkv_combine.  coff = N_k - N_q (causal: query i sees keys
// j <= i + coff).  Dense launches use {N, 0, 1, ceil(N / 128), null, null}.
struct SplitKv {
  int Nk, coff, n_split, kt_per;
  float* part_o;
  float* part_lse;
};

// --- bf16 tensor-core path (fa_fwd_sm100.cu, fa_bwd_sm100.cu) -------------
// Tensor maps describe a [BH, N, d] bf16 tensor as 3-D {d, N, BH} with a
// {64, 128, 1} box (loads) or a {64, 32, 1} box (the forward's O stores,
// `to`) and 128-byte swizzle.
constexpr int kStoreBoxRows = 32;
cudaError_t launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, void* o, float* lse, int BH, int N, int d,
                             float scale, int causal, const BlockMaskArg* bm, const Launch& L);

// Forward with 64-key tiles and two score buffers per query tile
// (fa_fwd64_sm100.cu); tk and tv have {64, 64, 1} boxes, tq {64, 128, 1},
// to {64, 32, 1}.  Dense only (no block mask, no split).
cudaError_t launch_fwd64_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& to, float* lse, int BH, int N, int d,
                               float scale, int causal, const Launch& L);

// Split-KV forward: tq has N_q rows per head, tk / tv N_k (sk.Nk) rows.
cudaError_t launch_fwd_splitkv_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                     const CUtensorMap& tv, int BH, int Nq, int d, float scale,
                                     int causal, const SplitKv& sk, const Launch& L);

// Merge of the split-KV partials: LSE = m + ln sum_s e^(LSE_s - m),
// O = sum_s e^(LSE_s - LSE) O_s (bf16 out); rows with every LSE_s = -inf give
// O = 0, LSE = -inf.  rows = BH * N_q.
cudaError_t launch_splitkv_combine(const float* part_o, const float* part_lse, void* o,
                                   float* lse, int n_split, int rows, int d, const Launch& L);

// Backward: the row-statistics kernel, the dQ kernel, then the dK/dV kernel,
// in stream order.  The first computes D = rowsum(dO o O) and LSE2 =
// LSE log2(e) from o, dO (bf16 [BH, N, d]) and lse into dvec and lse2
// ([BH, Np] fp32, Np = N rounded up to 128; D = 0 and LSE2 = +inf past N),
// which the other two read; dq, dk, dv are bf16 [BH, N, d] outputs.
cudaError_t launch_bwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const void* o, const void* dO,
                             const float* lse, float* dvec, float* lse2, void* dq, void* dk,
                             void* dv, int BH, int N, int d, float scale, int causal,
                             const BlockMaskArg* bm, const Launch& L);

// --- fp32 path helper (fa_simt.cu) -----------------------------------------
// D = rowsum(dO o O) (fp32, padded rows = 0) and, when lse2 is non-null,
// lse2 = LSE * log2(e) (padded rows = +inf).
cudaError_t launch_bwd_preprocess(const void* o, const void* dO, const float* lse, float* dvec,
                                  float* lse2, int BH, int N, int d, int is_bf16,
                                  const Launch& L);

// --- fp32 SIMT path (fa_simt.cu) -------------------------------------------
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int BH, int N, int d, float scale, int causal, const Launch& L);
cudaError_t launch_bwd_f32(const float* q, const float* k, const float* v, const float* dO,
                           const float* lse, const float* dvec, float* dq, float* dk, float* dv,
                           int BH, int N, int d, float scale, int causal, const Launch& L);

cudaError_t launch_selftest_wait(const Launch& L);

}  // namespace fa
