"""fp64 CPU oracle for the FP8 attention forward.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the
smoke check and the benchmark's baseline legs may use it; it shares no code
with the CUDA path.

What it computes, and where the pages define it
-----------------------------------------------
The FlashAttention-2 review page names FP8 as the piece FlashAttention-2
lacks (limitations, item 4) and, under future work, (5) "FP8 and latest
hardware", asks for FP8 in both the matmuls and the softmax; the auto-tuning
answer, section 1 (2), adds that FP8, FP16 and FP32 are to be mixed to keep
accuracy.  The pages fix no FP8 format, scaling or rounding.  Readings used:

* Q, K and V are stored as E4M3 codes: 1 sign bit, 4 exponent bits with
  bias 7, 3 mantissa bits, subnormals (exponent field 0: value
  mantissa / 8 * 2^-6), no infinities, and the all-ones exponent-and-mantissa
  pattern (0x7F, 0xFF) is NaN, so the largest finite value is
  1.75 * 2^8 = 448.  Each tensor carries one fp32 dequantisation factor
  (``descale``): element e stands for e4m3(code_e) * descale.
* The FP8 path approximates the exact attention of those dequantised inputs,
  so ``forward`` is the dense definition (``oracle.attention_forward``) on
  them, in fp64.
* The FP8 path also rounds the probabilities P to E4M3 before the P V product
  (the softmax in FP8); the running maximum it rounds them against is the
  kernel's, so the oracle does not try to reproduce that rounding.
  ``p_rounding_bound`` bounds, per output element, how far it can move the
  result, computed from the exact P.

The bound.  A probability p > 0 (relative to a reference maximum m <= the
row's true maximum M, so p = c P~ with P~ = exp(s - M) and c >= 1) rounds to
the nearest E4M3 value.  For p >= 2^-6 (normal range) the error is at most
half a unit in the last place, 2^-4 p; below 2^-6 (subnormal spacing 2^-9)
it is at most min(p, 2^-10).  The path divides the sum of rounded p v by the
fp32 sum of the unrounded p, l = c L~ with L~ = sum_j P~_j, so the rounding
moves O_ic by at most
    sum_j |v_jc| max(2^-4 P_ij, min(P_ij, 2^-10 / L~_i)),
with P the exact softmax (the factor c >= 1 only shrinks the subnormal term).
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .attention import _heads, as_f64, attention_forward, scores

E4M3_MAX = 448.0
E4M3_REL_HALF_ULP = 2.0 ** -4   # normal range: |RN(x) - x| <= 2^-4 |x|
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUB_HALF_SPACING = 2.0 ** -10


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code (uint8 array or torch uint8 tensor), float64;
    NaN for 0x7F and 0xFF."""
    if hasattr(codes, "detach"):
        codes = codes.detach().cpu().numpy()
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    val = sign * np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def dequantize(codes, descale: float) -> np.ndarray:
    """e4m3(code) * descale, float64 (descale is the tensor's fp32 factor)."""
    return e4m3_decode(codes) * float(np.float32(descale))


def forward(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float,
            scale: float, causal: bool = False,
            workers: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """O and LSE of exact attention on the dequantised FP8 inputs, fp64.

    q8, k8, v8: E4M3 codes [..., N, d] (uint8); the descale factors are the
    per-tensor fp32 dequantisation factors.  Returns O [..., N, d] and LSE
    [..., N] (natural log)."""
    q = dequantize(q8, q_descale)
    k = dequantize(k8, k_descale)
    v = dequantize(v8, v_descale)
    return attention_forward(q, k, v, scale, causal, workers=workers)


def p_rounding_bound(q, k, v, scale: float, causal: bool = False,
                     row_chunk: int = 1024) -> np.ndarray:
    """Per-element bound [..., N, d] on how far rounding the probabilities to
    E4M3 can move O (the formula in the module docstring), for dequantised
    fp64 inputs q, k, v [..., N, d]."""
    qh, lead = _heads(as_f64(q))
    kh, _ = _heads(as_f64(k))
    vh, _ = _heads(as_f64(v))
    n = qh.shape[1]
    out = np.empty(qh.shape[:2] + (vh.shape[2],), dtype=np.float64)
    for g in range(qh.shape[0]):
        av = np.abs(vh[g])
        for r0 in range(0, n, row_chunk):
            r1 = min(n, r0 + row_chunk)
            s = scores(qh[g, r0:r1], kh[g], scale, causal, r0)
            e = np.exp(s - np.max(s, axis=1, keepdims=True))   # P~, in (0, 1]
            lt = np.sum(e, axis=1, keepdims=True)              # L~
            p = e / lt
            w = np.maximum(E4M3_REL_HALF_ULP * p,
                           np.minimum(p, E4M3_SUB_HALF_SPACING / lt))
            out[g, r0:r1] = w @ av
    return out.reshape(lead + out.shape[1:])
