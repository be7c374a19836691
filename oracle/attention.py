"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, the smoke check and the benchmark's
``cpu_baseline`` / ``--impl reference`` legs use it.  It shares no code with
the CUDA path (no kernels, headers, helpers or constants); the only thing both
sides share is the seeded input generator in ``workloads``.

What it computes, and where the pages define it
-----------------------------------------------
* Standard attention in three steps, S = Q K^T, P = softmax(S), O = P V
  ("FlashAttention-2: Faster Attention with Better Parallelism and Work
  Partitioning" review, core-algorithm answer, section 1 "basic operation";
  "IO-4 FlashAttention" note, section 1 "Standard Attention memory flow").
* The scaled form softmax(Q K^T / sqrt(d_k)) V ("IO-4 FlashAttention", the
  problem statement; "Flash Attention-3" post, the code example, which scales
  by d ** -0.5).  ``scale`` is an argument here.
* Causal masking is not on the pages.  Reading used: query i sees keys
  j <= i (square problem), masked probabilities are exactly zero.
* The saved row statistic: the pages keep the running max m and running sum
  l ("FlashAttention-2" review, core-algorithm answer, (2) forward pass, step
  2 online softmax, and (3) backward pass, step 1).  The oracle returns the
  single natural-log value LSE = m + ln(l), which carries the same
  information.
* The backward: dV = P^T dO, dP = dO V^T, dS the softmax Jacobian applied to
  dP, dQ = dS K, dK = dS^T Q ("FlashAttention-2" review, (3) backward pass,
  step 2).  The page prints dS as "dP.P - P.(dP.P^T)" and leaves the scale
  out; the reading used is the row-wise Jacobian dS = P o (dP - rowsum(P o
  dP)) and dQ = scale dS K, dK = scale dS^T Q (chain rule through
  S = scale Q K^T).

``online_softmax_forward`` restates the blocked algorithm of the same pages
(tiles Q_i of B_r rows and K_j, V_j of B_c rows, a running max and a running
sum, one final normalisation).  It exists so the tests can show that the
blocked recurrence, with the carry term e^(m_old - m_new) the page's
l-formula omits, reproduces the full softmax; the GPU parity tests compare
against ``attention_forward`` / ``attention_backward``.

Everything is float64 numpy.  Inputs may be any float dtype (bf16 inputs are
torch tensors or numpy float32 copies of the bf16 values); they are widened to
float64 exactly before any arithmetic.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Tuple

import numpy as np

# Query rows handled per chunk: full key rows are kept, so a chunk's score
# block is chunk x N doubles (1024 x 16384 x 8 B = 128 MB at the longest
# workload).  Chunking rows changes nothing in the result: every row's
# softmax is still taken over all of its keys at once.
ROW_CHUNK = 1024


def as_f64(x) -> np.ndarray:
    """Widen a numpy array or torch tensor (any float dtype) to float64."""
    if hasattr(x, "detach"):            # torch tensor
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


def _heads(x: np.ndarray) -> Tuple[np.ndarray, Tuple[int, ...]]:
    """View [..., N, d] as [G, N, d] with G = product of leading dims."""
    lead = x.shape[:-2]
    return x.reshape((-1,) + x.shape[-2:]), lead


def scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
           row0: int = 0) -> np.ndarray:
    """S = scale * Q K^T for one head, with -inf where the causal mask hides
    key j from query i (j > i).  ``q`` holds query rows row0.. of the head."""
    s = scale * (q @ k.T)
    if causal:
        qi = np.arange(row0, row0 + q.shape[0])[:, None]
        kj = np.arange(k.shape[0])[None, :]
        s = np.where(kj > qi, -np.inf, s)
    return s


def softmax_rows(s: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Row softmax of a score block and its natural-log normaliser.

    Returns (P, lse) with P = exp(S - m) / l and lse = m + ln(l), where
    m = rowmax(S) and l = rowsum(exp(S - m)).
    """
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def _forward_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                  causal: bool) -> Tuple[np.ndarray, np.ndarray]:
    n = q.shape[0]
    o = np.empty((n, v.shape[1]), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    for r0 in range(0, n, ROW_CHUNK):
        r1 = min(n, r0 + ROW_CHUNK)
        p, l = softmax_rows(scores(q[r0:r1], k, scale, causal, r0))
        o[r0:r1] = p @ v
        lse[r0:r1] = l
    return o, lse


def _pool(workers: Optional[int]) -> int:
    return workers if workers else (os.cpu_count() or 1)


def attention_forward(q, k, v, scale: float, causal: bool = False,
                      workers: Optional[int] = None
                      ) -> Tuple[np.ndarray, np.ndarray]:
    """O = softmax(scale Q K^T [+ causal mask]) V and LSE, per head, fp64.

    q, k, v: [..., N, d] (any leading dims, e.g. [B, H, N, d]).
    Returns O [..., N, d] and LSE [..., N] (natural log) as float64.
    Heads are independent; a thread pool spreads them over the host cores
    (numpy releases the GIL in matmul and exp).
    """
    q, lead = _heads(as_f64(q))
    k, _ = _heads(as_f64(k))
    v, _ = _heads(as_f64(v))
    g = q.shape[0]
    o = np.empty(q.shape[:2] + (v.shape[2],), dtype=np.float64)
    lse = np.empty(q.shape[:2], dtype=np.float64)

    def one(h):
        o[h], lse[h] = _forward_head(q[h], k[h], v[h], scale, causal)

    nw = min(_pool(workers), g)
    if nw <= 1:
        for h in range(g):
            one(h)
    else:
        with ThreadPoolExecutor(nw) as ex:
            list(ex.map(one, range(g)))
    return o.reshape(lead + o.shape[1:]), lse.reshape(lead + lse.shape[1:])


def attention_probs(q, k, scale: float, causal: bool = False) -> np.ndarray:
    """The full probability matrix P [..., N, N] (small cases only)."""
    q, lead = _heads(as_f64(q))
    k, _ = _heads(as_f64(k))
    p = np.stack([softmax_rows(scores(q[h], k[h], scale, causal))[0]
                  for h in range(q.shape[0])])
    return p.reshape(lead + p.shape[1:])


def _backward_head(q, k, v, do, scale, causal, want_ds):
    n = q.shape[0]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    ds_full = np.empty((n, k.shape[0])) if want_ds else None
    dvec = np.empty(n)
    for r0 in range(0, n, ROW_CHUNK):
        r1 = min(n, r0 + ROW_CHUNK)
        p, _ = softmax_rows(scores(q[r0:r1], k, scale, causal, r0))
        dp = do[r0:r1] @ v.T                       # dP = dO V^T
        dd = np.sum(p * dp, axis=1, keepdims=True)  # rowsum(P o dP)
        ds = p * (dp - dd)                          # softmax Jacobian
        dv += p.T @ do[r0:r1]                       # dV = P^T dO
        dq[r0:r1] = scale * (ds @ k)                # dQ = scale dS K
        dk += scale * (ds.T @ q[r0:r1])             # dK = scale dS^T Q
        dvec[r0:r1] = dd[:, 0]
        if want_ds:
            ds_full[r0:r1] = ds
    return dq, dk, dv, dvec, ds_full


def attention_backward(q, k, v, do, scale: float, causal: bool = False,
                       workers: Optional[int] = None, return_aux: bool = False):
    """Gradients of O = attention(Q, K, V) for an upstream gradient dO, fp64.

    P is recomputed from Q and K (nothing from the forward is reused), then
    dV = P^T dO, dP = dO V^T, D = rowsum(P o dP), dS = P o (dP - D),
    dQ = scale dS K, dK = scale dS^T Q.

    Returns (dq, dk, dv), and with ``return_aux`` also (D, dS) where D is
    [..., N] and dS is [..., N, N] (small cases only).
    """
    q, lead = _heads(as_f64(q))
    k, _ = _heads(as_f64(k))
    v, _ = _heads(as_f64(v))
    do, _ = _heads(as_f64(do))
    g = q.shape[0]
    res = [None] * g

    def one(h):
        res[h] = _backward_head(q[h], k[h], v[h], do[h], scale, causal,
                                return_aux)

    nw = min(_pool(workers), g)
    if nw <= 1:
        for h in range(g):
            one(h)
    else:
        with ThreadPoolExecutor(nw) as ex:
            list(ex.map(one, range(g)))
    dq = np.stack([r[0] for r in res]).reshape(lead + q.shape[1:])
    dk = np.stack([r[1] for r in res]).reshape(lead + k.shape[1:])
    dv = np.stack([r[2] for r in res]).reshape(lead + v.shape[1:])
    if not return_aux:
        return dq, dk, dv
    dvec = np.stack([r[3] for r in res]).reshape(lead + q.shape[1:2])
    ds = np.stack([r[4] for r in res]).reshape(lead + (q.shape[1], k.shape[1]))
    return dq, dk, dv, dvec, ds


def online_softmax_forward(q, k, v, scale: float, causal: bool,
                           block_r: int, block_c: int,
                           kv_order=None) -> Tuple[np.ndarray, np.ndarray]:
    """The blocked forward with a running max and running sum, one head.

    Follows the pages' steps: split Q into row blocks Q_i of ``block_r``
    rows and K, V into blocks K_j, V_j of ``block_c`` rows; for each Q_i
    visit the K/V blocks, form S_ij = scale Q_i K_j^T, update the running
    max m = max(m, rowmax S_ij), carry the running sum and the unnormalised
    output with the factor e^(m_old - m_new), add exp(S_ij - m) and
    exp(S_ij - m) V_j, and divide by the running sum once at the end
    ("FlashAttention-2" review, core-algorithm answer, (1) tiling and (2)
    forward pass; the deferred division is the FA2 change listed under
    "original points", minimising non-matmul work).  ``kv_order`` visits the
    K/V blocks in a given order (the merge is order-independent).

    q, k, v: [N, d] for a single head.  Returns (O, LSE).
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    n, nk = q.shape[0], k.shape[0]
    t_c = (nk + block_c - 1) // block_c
    order = list(range(t_c)) if kv_order is None else list(kv_order)
    o = np.empty((n, v.shape[1]))
    lse = np.empty(n)
    for r0 in range(0, n, block_r):
        r1 = min(n, r0 + block_r)
        m = np.full(r1 - r0, -np.inf)
        l = np.zeros(r1 - r0)
        acc = np.zeros((r1 - r0, v.shape[1]))
        for j in order:
            c0, c1 = j * block_c, min(nk, (j + 1) * block_c)
            s = scale * (q[r0:r1] @ k[c0:c1].T)
            if causal:
                qi = np.arange(r0, r1)[:, None]
                kj = np.arange(c0, c1)[None, :]
                s = np.where(kj > qi, -np.inf, s)
            m_new = np.maximum(m, np.max(s, axis=1))
            # rows whose keys so far are all masked keep m = -inf; use 0
            # as the reference there so no (-inf) - (-inf) appears.
            ref = np.where(np.isfinite(m_new), m_new, 0.0)
            carry = np.exp(np.where(np.isfinite(m), m - ref, -np.inf))
            p = np.exp(s - ref[:, None])
            l = carry * l + np.sum(p, axis=1)
            acc = carry[:, None] * acc + p @ v[c0:c1]
            m = m_new
        o[r0:r1] = acc / l[:, None]
        lse[r0:r1] = m + np.log(l)
    return o, lse


def printed_block_sum_forward(q, k, v, scale: float, block_c: int
                              ) -> np.ndarray:
    """The tiled formula exactly as the "IO-4 FlashAttention" note prints it
    (section 3, "O_i = sum_j softmax(Q_i K_j^T) V_j": a separate softmax per
    key block, summed, with no rescaling).  Kept only so a test can show that
    this printed form is NOT attention; it is never used as a reference."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    out = np.zeros((q.shape[0], v.shape[1]))
    for c0 in range(0, k.shape[0], block_c):
        c1 = min(k.shape[0], c0 + block_c)
        p, _ = softmax_rows(scale * (q @ k[c0:c1].T))
        out += p @ v[c0:c1]
    return out
