"""fp64 CPU oracle for block-sparse attention.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the
smoke check and the benchmark's baseline legs may use it; it shares no code
with the CUDA path.

What it computes, and where the pages define it
-----------------------------------------------
Block-sparse FlashAttention is the combination the "FlashAttention-2: Faster
Attention with Better Parallelism and Work Partitioning" review describes in
its answer on joining FlashAttention-2 with sparse or hybrid attention,
section 3 (1) "Sparse FlashAttention": a sparsity pattern defined on blocks
(e.g. local context), matched to the kernel's tile sizes, and only the
important blocks processed on chip; its limitations answer, section 2 (3),
adds the hybrid form (dense global attention plus sparse local attention).
The pages give no formula beyond that, so the reading used is the plain one:

* ``block_mask[h, I, J]`` (bool) says whether query block I of head h may
  attend to key block J; blocks are ``block`` x ``block`` squares of the
  N x N score matrix (the last block row/column may be ragged).
* The score matrix is the dense one, S = scale Q K^T, with -inf wherever the
  block mask (and, with ``causal``, the causal mask j > i) hides a key; the
  result is the softmax of those scores, i.e. the dense definition of
  ``oracle.attention`` with the hidden entries removed.
* A query row that sees no key at all has no softmax; the reading used is
  O = 0 and LSE = -inf for that row, and it contributes nothing to any
  gradient (dQ row = 0).

A mask with one head (shape [1, nb, nb] or [nb, nb]) applies to every head;
otherwise it has H heads and head h of every batch entry uses block_mask[h].
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

from .attention import as_f64


def n_blocks(n: int, block: int) -> int:
    return (n + block - 1) // block


def _mask_heads(block_mask) -> np.ndarray:
    m = np.asarray(block_mask).astype(bool)
    if m.ndim == 2:
        m = m[None]
    if m.ndim != 3 or m.shape[1] != m.shape[2]:
        raise ValueError("block_mask must be [nb, nb] or [Hm, nb, nb]")
    return m


def element_mask(block_mask_h: np.ndarray, n: int, block: int, causal: bool) -> np.ndarray:
    """[N, N] bool: True where query i may attend to key j."""
    nb = n_blocks(n, block)
    if block_mask_h.shape != (nb, nb):
        raise ValueError(f"block mask is {block_mask_h.shape}, expected {(nb, nb)}")
    bi = np.arange(n) // block
    allowed = block_mask_h[bi[:, None], bi[None, :]]
    if causal:
        allowed = allowed & (np.arange(n)[None, :] <= np.arange(n)[:, None])
    return allowed


def _probs(q, k, scale, allowed):
    """P (rows with no visible key are all zero) and LSE (-inf there)."""
    s = np.where(allowed, scale * (q @ k.T), -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.where(allowed, np.exp(s - m_safe), 0.0)
    l = np.sum(e, axis=1, keepdims=True)
    p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
    lse = np.where(empty, -np.inf, (m_safe + np.log(np.where(l > 0, l, 1.0)))[:, 0])
    return p, lse


def _per_head(x):
    x = as_f64(x)
    return x.reshape((-1,) + x.shape[-2:]), x.shape[:-2]


def block_sparse_forward(q, k, v, scale: float, block_mask, causal: bool = False,
                         block: int = 128) -> Tuple[np.ndarray, np.ndarray]:
    """O and LSE (natural log) of block-sparse attention, fp64.

    q, k, v: [B, H, N, d] (or [H, N, d] / [N, d]); block_mask as described in
    the module docstring.  Returns O [..., N, d] and LSE [..., N].
    """
    qh, lead = _per_head(q)
    kh, _ = _per_head(k)
    vh, _ = _per_head(v)
    m = _mask_heads(block_mask)
    H = lead[-1] if len(lead) >= 1 else 1
    n = qh.shape[1]
    o = np.zeros(qh.shape[:2] + (vh.shape[2],))
    lse = np.empty(qh.shape[:2])
    for g in range(qh.shape[0]):
        mh = m[0] if m.shape[0] == 1 else m[g % H]
        allowed = element_mask(mh, n, block, causal)
        p, lse[g] = _probs(qh[g], kh[g], scale, allowed)
        o[g] = p @ vh[g]
    return o.reshape(lead + o.shape[1:]), lse.reshape(lead + lse.shape[1:])


def block_sparse_backward(q, k, v, do, scale: float, block_mask, causal: bool = False,
                          block: int = 128):
    """dQ, dK, dV of block-sparse attention for upstream gradient dO, fp64.

    The same formulas as the dense oracle on the masked P:
    dV = P^T dO, dP = dO V^T, dS = P o (dP - rowsum(P o dP)),
    dQ = scale dS K, dK = scale dS^T Q.  Hidden entries have P = 0, hence
    dS = 0; a row with no visible key gets dQ = 0.
    """
    qh, lead = _per_head(q)
    kh, _ = _per_head(k)
    vh, _ = _per_head(v)
    doh, _ = _per_head(do)
    m = _mask_heads(block_mask)
    H = lead[-1] if len(lead) >= 1 else 1
    n = qh.shape[1]
    dq = np.zeros_like(qh)
    dk = np.zeros_like(kh)
    dv = np.zeros_like(vh)
    for g in range(qh.shape[0]):
        mh = m[0] if m.shape[0] == 1 else m[g % H]
        allowed = element_mask(mh, n, block, causal)
        p, _ = _probs(qh[g], kh[g], scale, allowed)
        dp = doh[g] @ vh[g].T
        ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
        dv[g] = p.T @ doh[g]
        dq[g] = scale * (ds @ kh[g])
        dk[g] = scale * (ds.T @ qh[g])
    shape = lambda x: x.reshape(lead + x.shape[1:])
    return shape(dq), shape(dk), shape(dv)


def brute_forward(q, k, v, scale: float, block_mask_h, causal: bool, block: int):
    """Scalar loops for one head (tiny N only): the definition written out
    element by element, independent of the vectorised code above."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    n, d = q.shape
    o = np.zeros((n, v.shape[1]))
    lse = np.empty(n)
    for i in range(n):
        keys = [j for j in range(n)
                if block_mask_h[i // block][j // block] and (not causal or j <= i)]
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
