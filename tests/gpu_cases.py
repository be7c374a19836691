"""Shared helpers for the GPU parity tests: run the library through its C ABI
on seeded inputs and compare with the fp64 oracle on the same bits."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

# Tolerances (forward O and LSE, gradients relative to the largest reference
# magnitude of each tensor).
TOL_O_BF16 = 1e-2
TOL_O_FP32 = 1e-5
TOL_LSE = 1e-3
TOL_GRAD_REL = 2e-2
# When a gradient is identically zero in exact arithmetic (N = 1: the softmax
# over one key is constant, so dQ = dK = 0) the relative bound would demand
# bit-exact zeros from two differently ordered fp32 sums; the reference
# magnitude is floored at this value instead (an absolute bound of 2e-6).
GRAD_REF_FLOOR = 1e-4


def fa():
    import exact_io_aware_99_b200 as m
    return m


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().cuda()


def gpu_forward(q, k, v, scale, causal):
    m = fa()
    B, H, N, d = q.shape
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    dt = m.FA_FP32 if q.dtype == torch.float32 else m.FA_BF16
    m.fa_forward_ex(qd, kd, vd, o, lse, B, H, N, d, scale, causal, dt)
    torch.cuda.synchronize()
    st, site = m.fa_device_status(reset=True)
    assert st == 0, f"device wait timed out at site {site:#x}"
    return o, lse


def gpu_backward(q, k, v, o, do, lse, scale, causal):
    m = fa()
    B, H, N, d = q.shape
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    od = o if o.is_cuda else to_dev(o)
    lsed = lse if lse.is_cuda else to_dev(lse)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    wb = m.fa_backward_workspace_size(B, H, N, d)
    ws = torch.empty(wb, device="cuda", dtype=torch.uint8)
    dt = m.FA_FP32 if q.dtype == torch.float32 else m.FA_BF16
    m.fa_backward_ex(qd, kd, vd, od, dod, lsed, dq, dk, dv, B, H, N, d, scale, causal, ws, wb, dt)
    torch.cuda.synchronize()
    st, site = m.fa_device_status(reset=True)
    assert st == 0, f"device wait timed out at site {site:#x}"
    return dq, dk, dv


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_forward(q, k, v, scale, causal, heads=None, tol_o=None):
    """GPU forward vs oracle.  ``heads``: list of (b, h) to compare (all when
    None); the GPU always runs the whole problem."""
    o, lse = gpu_forward(q, k, v, scale, causal)
    tol_o = tol_o if tol_o is not None else (TOL_O_FP32 if q.dtype == torch.float32
                                             else TOL_O_BF16)
    B, H = q.shape[:2]
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    worst_o = worst_l = 0.0
    for b, h in pairs:
        ro, rl = oracle.attention_forward(q[b, h], k[b, h], v[b, h], scale, causal)
        go, gl = np64(o[b, h]), np64(lse[b, h])
        assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
        worst_o = max(worst_o, float(np.max(np.abs(go - ro))))
        worst_l = max(worst_l, float(np.max(np.abs(gl - rl))))
    assert worst_o <= tol_o, f"O max abs err {worst_o:.3g} > {tol_o}"
    assert worst_l <= TOL_LSE, f"LSE max abs err {worst_l:.3g} > {TOL_LSE}"
    return o, lse, worst_o, worst_l


def check_backward(q, k, v, do, scale, causal, heads=None):
    o, lse = gpu_forward(q, k, v, scale, causal)
    dq, dk, dv = gpu_backward(q, k, v, o, do, lse, scale, causal)
    B, H = q.shape[:2]
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    worst = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    for b, h in pairs:
        rq, rk, rv = oracle.attention_backward(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal)
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            gg = np64(g[b, h])
            assert np.all(np.isfinite(gg)), name
            err = float(np.max(np.abs(gg - r))) / max(float(np.max(np.abs(r))), GRAD_REF_FLOOR)
            worst[name] = max(worst[name], err)
    for name, err in worst.items():
        assert err <= TOL_GRAD_REL, f"{name} max abs err / max|ref| = {err:.3g} > {TOL_GRAD_REL}"
    return worst


def l2_group_heads(B, H, N, d, causal, kv_bytes=2):
    """(b, h) pairs a work-order mistake of the persistent kernels would hit
    first.  The kernels run heads in groups sized so that a group's K and V
    (2 N d elements of kv_bytes each per head) fit a 64 MB (causal) or 32 MB
    (non-causal) share of L2, group after group; a CTA takes further items
    by cancelling CTAs that have not started, so the first head of each
    group (where one group's items hand over to the next) and the whole last
    group (the items taken over at the end of the launch) are the ones to
    check.  Returned sorted, as (b, h) with bh = b H + h."""
    BH = B * H
    per_head = 2 * N * d * kv_bytes
    share = (64 if causal else 32) << 20
    g = max(1, min(BH, share // max(per_head, 1)))
    picks = set(range(0, BH, g))
    last = ((BH - 1) // g) * g
    picks.update(range(last, BH))
    return [divmod(bh, H) for bh in sorted(picks)]

