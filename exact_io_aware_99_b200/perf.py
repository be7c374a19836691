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
