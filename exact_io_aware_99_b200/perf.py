"""Algorithmic FLOP and byte counts for the attention workloads.

FLOPs follow the count on the "FlashAttention-2" review page (answer on
implementation cost, (1) FLOPs: forward 4 N^2 d per head, backward 2.5x the
forward; N = 1024, d = 64 gives 268,435,456 and 671,088,640), halved when
causal (only the j <= i half of the score matrix is work).

Bytes are what the method must move through HBM at minimum:
  forward   read Q, K, V; write O and the fp32 LSE.
  backward  read Q, K, V, O, dO and the LSE; write dQ, dK, dV.
"""
from __future__ import annotations


def fwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def bwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    return 2.5 * fwd_flops(B, H, N, d, causal)


def fwd_bytes(B: int, H: int, N: int, d: int, elem: int = 2) -> float:
    return 4.0 * B * H * N * d * elem + 4.0 * B * H * N


def bwd_bytes(B: int, H: int, N: int, d: int, elem: int = 2) -> float:
    return 8.0 * B * H * N * d * elem + 4.0 * B * H * N


def visible_pairs(block_mask, N: int, causal: bool, block: int = 128) -> float:
    """Number of (query, key) pairs a block mask (bool [Hm, nt, nt] or
    [nt, nt]) leaves visible, summed over its heads, with ragged edge tiles
    and the causal triangle counted exactly."""
    import numpy as np
    m = np.asarray(block_mask, dtype=bool)
    if m.ndim == 2:
        m = m[None]
    nt = m.shape[-1]
    size = np.full(nt, block, dtype=np.float64)
    size[-1] = N - block * (nt - 1)
    total = 0.0
    for i in range(nt):
        for j in range(nt):
            if causal and j > i:
                continue
            if causal and j == i:
                s = size[i]
                pairs = s * (s + 1) / 2
            else:
                pairs = size[i] * size[j]
            total += pairs * float(np.count_nonzero(m[:, i, j]))
    return total


def fwd_flops_masked(B: int, H: int, N: int, d: int, causal: bool, block_mask) -> float:
    """Forward FLOPs of block-sparse attention: 4 d per visible (query, key)
    pair (the dense count with only the visible pairs).  A per-head mask
    (H heads) is counted per head; a shared mask is counted H times."""
    import numpy as np
    m = np.asarray(block_mask, dtype=bool)
    heads = 1 if m.ndim == 2 else m.shape[0]
    pairs = visible_pairs(m, N, causal)
    per_batch = pairs * (H if heads == 1 else 1)
    return 4.0 * d * B * per_batch


def bwd_flops_masked(B: int, H: int, N: int, d: int, causal: bool, block_mask) -> float:
    return 2.5 * fwd_flops_masked(B, H, N, d, causal, block_mask)


def decode_pairs(Nq: int, Nk: int, causal: bool) -> float:
    """Visible (query, key) pairs of N_q queries that are the last N_q of N_k
    positions (causal: query i sees keys j <= i + N_k - N_q)."""
    if not causal:
        return float(Nq) * Nk
    total = 0.0
    for i in range(Nq):
        total += max(0, min(Nk, i + Nk - Nq + 1))
    return total


def decode_flops(B: int, H: int, Nq: int, Nk: int, d: int, causal: bool) -> float:
    return 4.0 * d * B * H * decode_pairs(Nq, Nk, causal)


def decode_bytes(B: int, H: int, Nq: int, Nk: int, d: int, elem: int = 2) -> float:
    """Q read + O written (N_q rows), K and V read (N_k rows), LSE written."""
    return 2.0 * B * H * Nq * d * elem + 2.0 * B * H * Nk * d * elem + 4.0 * B * H * Nq
