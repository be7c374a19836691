"""GPU parity for block-sparse attention (fa_forward_blocksparse /
fa_backward_blocksparse) against the block-sparse fp64 oracle on the same
seeded inputs: O, LSE (including the -inf of rows that see no key) and the
three gradients, with the bounds of the dense parity tests."""
import math

import numpy as np
import pytest
import torch

import workloads
from gpu_cases import GRAD_REF_FLOOR, TOL_GRAD_REL, TOL_LSE, TOL_O_BF16, np64
from oracle.block_sparse import block_sparse_backward, block_sparse_forward

pytestmark = pytest.mark.gpu

BLOCK = 128


def fa():
    import exact_io_aware_99_b200 as m
    return m


def random_mask(n_heads, nt, density, seed, empty_row=None, unseen_col=None):
    rs = np.random.default_rng(seed)
    m = rs.random((n_heads, nt, nt)) < density
    if empty_row is not None:
        m[:, empty_row, :] = False
    if unseen_col is not None:
        m[:, :, unseen_col] = False
    return m


def band_mask(nt, width, global_cols=()):
    i = np.arange(nt)
    m = np.abs(i[:, None] - i[None, :]) <= width
    for c in global_cols:
        m[:, c] = True
    return m[None]


def run_case(B, H, N, d, causal, mask, seed):
    m = fa()
    x = workloads.random_case(B, H, N, d, seed)
    scale = 1 / math.sqrt(d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    bm = torch.from_numpy(mask.astype(np.uint8))
    o, lse = m.attention_forward(q, k, v, scale=scale, causal=causal, block_mask=bm)
    dq, dk, dv = m.attention_backward(q, k, v, o, do, lse, scale=scale, causal=causal,
                                      block_mask=bm)
    torch.cuda.synchronize()
    st, site = m.fa_device_status(reset=True)
    assert st == 0, f"device wait timed out at site {site:#x}"
    ro, rl = block_sparse_forward(x["q"], x["k"], x["v"], scale, mask, causal, BLOCK)
    rdq, rdk, rdv = block_sparse_backward(x["q"], x["k"], x["v"], x["do"], scale, mask, causal,
                                          BLOCK)
    go, gl = np64(o), np64(lse)
    assert np.all(np.isfinite(go))
    err_o = float(np.max(np.abs(go - ro)))
    assert err_o <= TOL_O_BF16, f"O max abs err {err_o:.3g}"
    # rows that see no key: exactly -inf on both sides
    np.testing.assert_array_equal(np.isneginf(gl), np.isneginf(rl))
    fin = np.isfinite(rl)
    if fin.any():
        err_l = float(np.max(np.abs(gl[fin] - rl[fin])))
        assert err_l <= TOL_LSE, f"LSE max abs err {err_l:.3g}"
    for name, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        gg = np64(g)
        assert np.all(np.isfinite(gg)), name
        bound = TOL_GRAD_REL * max(float(np.max(np.abs(r))), GRAD_REF_FLOOR)
        err = float(np.max(np.abs(gg - r)))
        assert err <= bound, f"{name}: max abs err {err:.3g} > {bound:.3g}"
    return rl


@pytest.mark.parametrize("causal", [False, True])
def test_ragged_random_mask_with_empty_row_and_unseen_keys(causal):
    # N = 300: tiles of 128, 128, 44 rows; query tile 1 sees nothing, key
    # tile 2 is seen by no query.
    mask = random_mask(1, 3, 0.7, 11, empty_row=1, unseen_col=2)
    mask[:, 0, 0] = mask[:, 2, 0] = True
    rl = run_case(1, 2, 300, 128, causal, mask, 901)
    assert np.all(np.isneginf(rl[..., 128:256]))


@pytest.mark.parametrize("d", [64, 80, 128])
def test_per_head_masks(d):
    B, H, N = 2, 3, 1000                 # 8 tiles, ragged last one
    nt = (N + BLOCK - 1) // BLOCK
    mask = random_mask(H, nt, 0.5, 20 + d)
    run_case(B, H, N, d, True, mask, 930 + d)


def test_band_with_global_columns_non_causal():
    nt = 9
    run_case(1, 4, 9 * 128 - 50, 128, False, band_mask(nt, 1, global_cols=(0,)), 955)


def test_all_blocks_on_matches_dense_path():
    # the block-sparse forward is the 128-key kernel with a mask: with every
    # block on it must reproduce the dense 128-key kernel bit for bit
    m = fa()
    x = workloads.random_case(1, 2, 513, 128, 960)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    nt = 5
    bm = torch.ones((nt, nt), dtype=torch.uint8)
    m.fa_set_forward_key_tile(128)
    try:
        for causal in (False, True):
            o1, l1 = m.attention_forward(q, k, v, causal=causal, block_mask=bm)
            o2, l2 = m.attention_forward(q, k, v, causal=causal)
            torch.cuda.synchronize()
            assert torch.equal(o1, o2) and torch.equal(l1, l2)
    finally:
        m.fa_set_forward_key_tile(0)


def test_everything_hidden_gives_zeros():
    mask = np.zeros((1, 1, 1), bool)
    rl = run_case(1, 2, 100, 64, False, mask, 970)
    assert np.all(np.isneginf(rl))


def test_bad_mask_arguments_are_rejected():
    m = fa()
    x = workloads.random_case(1, 2, 256, 64, 980)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 256), device="cuda", dtype=torch.float32)
    bm = torch.ones((3, 2, 2), dtype=torch.uint8, device="cuda")
    st = m.fa_forward_blocksparse(q, k, v, o, lse, 1, 2, 256, 64, 0.125, 0, bm, 3, check=False)
    assert st == m.FA_ERR_INVALID_ARG     # mask_heads must be 1 or H
    st = m.fa_forward_blocksparse(q, k, v, o, lse, 1, 2, 256, 64, 0.125, 0, None, 1,
                                  check=False)
    assert st == m.FA_ERR_INVALID_ARG     # null mask
