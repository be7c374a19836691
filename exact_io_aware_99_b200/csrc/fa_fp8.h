// fa_fp8.h -- launch interface of the FP8 (E4M3) forward and the per-tensor
// E4M3 quantiser (fa_fwd_fp8_sm100.cu), used by the C ABI in fa_api.cu.
// Not installed; not part of the public ABI.
#pragma once

#include <cstddef>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_internal.h"

namespace fa {

// Wait-site codes of the FP8 forward (recorded in the status word when one
// of its bounded waits runs out).
constexpr int kSiteFp8Producer = 0x301;
constexpr int kSiteFp8Mma = 0x302;
constexpr int kSiteFp8Softmax = 0x303;
constexpr int kSiteFp8Epilogue = 0x304;
constexpr int kSiteFp8Drain = 0x305;

// Tensor maps of the FP8 forward describe a [BH, N, d] E4M3 tensor (one byte
// per element) as 3-D {d, N, BH} with a {128, 128, 1} box and 128-byte
// swizzle: a whole 128-byte row per query or key, columns past d read as 0.
// The descale pointers are device fp32 scalars (nullptr = 1).
cudaError_t launch_fwd_fp8_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const float* q_descale,
                                 const float* k_descale, const float* v_descale, void* o,
                                 float* lse, int BH, int N, int d, float scale, int causal,
                                 const Launch& L);

// Per-tensor E4M3 quantisation of n elements (bf16 when is_bf16, else fp32):
// amax = max |x| (accumulated into *descale, which the caller has zeroed),
// codes = RN_satfinite(x * (448 / amax)), then *descale = amax / 448
// (1 when amax = 0).  Three launches in stream order.
cudaError_t launch_quantize_e4m3(const void* x, int is_bf16, size_t n, uint8_t* codes,
                                 float* descale, const Launch& L);

}  // namespace fa
