"""fp64 CPU oracle for attention with fewer queries than keys (decode).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the
smoke check and the benchmark's baseline legs may use it; it shares no code
with the CUDA path.

What it computes, and where the pages define it
-----------------------------------------------
Decoding appends a few new queries (N_q) to a long cached key/value sequence
(N_k >= N_q).  The attention itself is the same definition as
``oracle.attention`` -- O = softmax(scale Q K^T) V row by row, LSE the
natural-log normaliser -- on a rectangular N_q x N_k score matrix.

* Causal masking is not on the pages; with N_q < N_k the reading used is the
  one that makes the queries the last N_q positions of the sequence: query i
  sees keys j <= i + (N_k - N_q) (so the last query sees every key).  With
  N_q = N_k this is the square causal mask of ``oracle.attention``.
* A row that sees no key (only possible when N_k < N_q) gets O = 0 and
  LSE = -inf, as in ``oracle.block_sparse``.

``merge_partials`` restates how partial results over disjoint key sets
combine into the full one: the running-max / running-sum merge of the online
softmax ("FlashAttention-2: Faster Attention with Better Parallelism and Work
Partitioning" review, core-algorithm answer, (2) forward pass step 2, with
the carry term e^(m_old - m_new) written out), applied to whole partial
results the way the review's answer on FlashAttention's Split-K scheme
describes K and V split across workers whose intermediate results are then
combined.  The tests use it to pin ``rect_forward`` on key chunks; the GPU
parity tests compare against ``rect_forward`` directly.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from .attention import as_f64


def _heads(x):
    x = as_f64(x)
    return x.reshape((-1,) + x.shape[-2:]), x.shape[:-2]


def visible(nq: int, nk: int, causal: bool) -> np.ndarray:
    """[N_q, N_k] bool: query i may attend to key j."""
    if not causal:
        return np.ones((nq, nk), bool)
    return np.arange(nk)[None, :] <= np.arange(nq)[:, None] + (nk - nq)


def _one_head(q, k, v, scale, allowed):
    s = np.where(allowed, scale * (q @ k.T), -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(allowed, np.exp(s - m), 0.0)
    l = np.sum(e, axis=1, keepdims=True)
    lsafe = np.where(l > 0, l, 1.0)
    o = (e / lsafe) @ v
    lse = np.where(empty, -np.inf, (m + np.log(lsafe))[:, 0])
    return o, lse


def rect_forward(q, k, v, scale: float, causal: bool = False) -> Tuple[np.ndarray, np.ndarray]:
    """O [..., N_q, d] and LSE [..., N_q] for q [..., N_q, d] against k, v
    [..., N_k, d], fp64."""
    qh, lead = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    nq, nk = qh.shape[1], kh.shape[1]
    allowed = visible(nq, nk, causal)
    o = np.empty(qh.shape[:2] + (vh.shape[2],))
    lse = np.empty(qh.shape[:2])
    for g in range(qh.shape[0]):
        o[g], lse[g] = _one_head(qh[g], kh[g], vh[g], scale, allowed)
    return o.reshape(lead + o.shape[1:]), lse.reshape(lead + lse.shape[1:])


def chunk_forward(q, k, v, scale: float, causal: bool, k0: int, k1: int):
    """Partial result over keys [k0, k1) only (same causal rule, measured in
    the full key sequence): O normalised over those keys and their LSE
    (-inf where a row sees none of them)."""
    qh, lead = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    nq, nk = qh.shape[1], kh.shape[1]
    allowed = visible(nq, nk, causal)[:, k0:k1]
    o = np.empty(qh.shape[:2] + (vh.shape[2],))
    lse = np.empty(qh.shape[:2])
    for g in range(qh.shape[0]):
        o[g], lse[g] = _one_head(qh[g], kh[g, k0:k1], vh[g, k0:k1], scale, allowed)
    return o.reshape(lead + o.shape[1:]), lse.reshape(lead + lse.shape[1:])


def merge_partials(o_parts: Sequence[np.ndarray], lse_parts: Sequence[np.ndarray]):
    """Combine partial (O_s, LSE_s) over disjoint key sets:
    LSE = m + ln sum_s e^(LSE_s - m) with m = max_s LSE_s, and
    O = sum_s e^(LSE_s - LSE) O_s.  Rows with every LSE_s = -inf stay
    O = 0, LSE = -inf."""
    lse = np.stack([as_f64(x) for x in lse_parts])
    o = np.stack([as_f64(x) for x in o_parts])
    m = np.max(lse, axis=0)
    finite = np.isfinite(m)
    msafe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(lse), np.exp(lse - msafe), 0.0)
    tot = np.sum(w, axis=0)
    out_lse = np.where(finite, msafe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    wn = w / np.where(tot > 0, tot, 1.0)
    out_o = np.sum(wn[..., None] * o, axis=0)
    return out_o, out_lse


def brute_forward(q, k, v, scale: float, causal: bool):
    """Scalar loops for one head (tiny sizes only)."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    nq, nk, d = q.shape[0], k.shape[0], q.shape[1]
    o = np.zeros((nq, v.shape[1]))
    lse = np.empty(nq)
    for i in range(nq):
        keys = [j for j in range(nk) if not causal or j <= i + (nk - nq)]
        if not keys:
            lse[i] = -np.inf
            continue
        sc = [scale * sum(q[i, c] * k[j, c] for c in range(d)) for j in keys]
        mx = max(sc)
        w = [np.exp(x - mx) for x in sc]
        tot = sum(w)
        for t, j in enumerate(keys):
            o[i] += (w[t] / tot) * v[j]
        lse[i] = mx + np.log(tot)
    return o, lse
