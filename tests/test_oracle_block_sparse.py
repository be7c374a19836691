"""Pins for the block-sparse oracle (oracle/block_sparse.py), CPU only.

Each test ties the oracle to something other than itself: the dense oracle on
sub-problems the mask carves out, a scalar brute-force loop, finite
differences, and closed-form facts about fully hidden rows.  A plausible
mistake -- a transposed mask, a block index off by one, a missing -inf, a
gradient that leaks through hidden entries -- fails at least one of them.
"""
import numpy as np
import pytest

from oracle import attention_backward, attention_forward
from oracle.block_sparse import (block_sparse_backward, block_sparse_forward, brute_forward,
                                 element_mask, n_blocks)

RNG = np.random.default_rng(20260)


def rand(*shape):
    return RNG.standard_normal(shape)


@pytest.mark.parametrize("causal", [False, True])
def test_all_blocks_on_is_dense_attention(causal):
    q, k, v, do = (rand(2, 3, 37, 8) for _ in range(4))
    nb = n_blocks(37, 8)
    mask = np.ones((nb, nb), bool)
    o, lse = block_sparse_forward(q, k, v, 0.3, mask, causal, block=8)
    od, lsed = attention_forward(q, k, v, 0.3, causal)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lsed, rtol=0, atol=1e-12)
    g = block_sparse_backward(q, k, v, do, 0.3, mask, causal, block=8)
    gd = attention_backward(q, k, v, do, 0.3, causal)
    for a, b in zip(g, gd):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_block_diagonal_mask_is_independent_attention_per_block():
    n, blk = 20, 6                      # blocks 0-5, 6-11, 12-17, 18-19 (ragged)
    q, k, v = rand(n, 5), rand(n, 5), rand(n, 7)
    nb = n_blocks(n, blk)
    o, lse = block_sparse_forward(q, k, v, 0.7, np.eye(nb, dtype=bool), False, block=blk)
    for b in range(nb):
        sl = slice(b * blk, min(n, (b + 1) * blk))
        ob, lb = attention_forward(q[sl], k[sl], v[sl], 0.7, False)
        np.testing.assert_allclose(o[sl], ob, atol=1e-12)
        np.testing.assert_allclose(lse[sl], lb, atol=1e-12)


def test_each_query_block_sees_one_other_key_block():
    # Query block I sees only key block perm[I] (a 3-cycle, so a transposed
    # mask would pick perm^-1 and fail).
    n, blk = 12, 4
    perm = [1, 2, 0]
    mask = np.zeros((3, 3), bool)
    for i, j in enumerate(perm):
        mask[i, j] = True
    q, k, v = rand(n, 3), rand(n, 3), rand(n, 2)
    o, lse = block_sparse_forward(q, k, v, 1.1, mask, False, block=blk)
    for i, j in enumerate(perm):
        qs, ks = slice(i * blk, (i + 1) * blk), slice(j * blk, (j + 1) * blk)
        ob, lb = attention_forward(q[qs], k[ks], v[ks], 1.1, False)
        np.testing.assert_allclose(o[qs], ob, atol=1e-12)
        np.testing.assert_allclose(lse[qs], lb, atol=1e-12)


def test_hidden_rows_give_zero_output_minus_inf_lse_and_no_gradient():
    n, blk = 10, 4                       # blocks 0-3, 4-7, 8-9
    mask = np.array([[1, 0, 0], [0, 0, 0], [1, 0, 1]], bool)   # query block 1 sees nothing
    q, k, v, do = rand(n, 3), rand(n, 3), rand(n, 3), rand(n, 3)
    o, lse = block_sparse_forward(q, k, v, 0.5, mask, False, block=blk)
    np.testing.assert_array_equal(o[4:8], 0.0)
    assert np.all(np.isneginf(lse[4:8])) and np.all(np.isfinite(lse[[0, 1, 2, 3, 8, 9]]))
    dq, dk, dv = block_sparse_backward(q, k, v, do, 0.5, mask, False, block=blk)
    np.testing.assert_array_equal(dq[4:8], 0.0)
    # dK and dV do not depend on the hidden rows' queries or upstream gradients
    q2, do2 = q.copy(), do.copy()
    q2[4:8] = rand(4, 3)
    do2[4:8] = rand(4, 3)
    _, dk2, dv2 = block_sparse_backward(q2, k, v, do2, 0.5, mask, False, block=blk)
    np.testing.assert_allclose(dk2, dk, atol=1e-14)
    np.testing.assert_allclose(dv2, dv, atol=1e-14)
    # key block 1 is seen by no query: its gradients are exactly zero
    np.testing.assert_array_equal(dk[4:8], 0.0)
    np.testing.assert_array_equal(dv[4:8], 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_vectorised_oracle_matches_scalar_loops(causal):
    n, blk = 9, 2
    nb = n_blocks(n, blk)
    mask = RNG.random((nb, nb)) < 0.5
    mask[2, :] = False                   # one empty query block
    q, k, v = rand(n, 3), rand(n, 3), rand(n, 4)
    o, lse = block_sparse_forward(q, k, v, 0.8, mask, causal, block=blk)
    ob, lb = brute_forward(q, k, v, 0.8, mask, causal, blk)
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], atol=1e-12)


def test_per_head_masks_pick_head_h_for_every_batch_entry():
    B, H, n, blk = 2, 3, 8, 4
    masks = RNG.random((H, 2, 2)) < 0.6
    masks[:, :, 0] = True                # every query block sees key block 0
    q, k, v = rand(B, H, n, 3), rand(B, H, n, 3), rand(B, H, n, 3)
    o, lse = block_sparse_forward(q, k, v, 0.4, masks, False, block=blk)
    for b in range(B):
        for h in range(H):
            oh, lh = block_sparse_forward(q[b, h], k[b, h], v[b, h], 0.4, masks[h], False,
                                          block=blk)
            np.testing.assert_allclose(o[b, h], oh, atol=1e-13)
            np.testing.assert_allclose(lse[b, h], lh, atol=1e-13)


def test_gradients_match_central_finite_differences():
    n, blk, d = 6, 2, 3
    mask = np.array([[1, 0, 0], [1, 1, 0], [0, 1, 1]], bool)
    q, k, v, do = rand(n, d), rand(n, d), rand(n, d), rand(n, d)
    scale = 0.9
    for causal in (False, True):
        dq, dk, dv = block_sparse_backward(q, k, v, do, scale, mask, causal, block=blk)

        def loss(qq, kk, vv):
            o, _ = block_sparse_forward(qq, kk, vv, scale, mask, causal, block=blk)
            return float(np.sum(o * do))

        h = 1e-6
        for arr, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
            num = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[which][idx] += h
                args_m[which][idx] -= h
                num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            err = np.max(np.abs(num - grad)) / max(np.max(np.abs(grad)), 1e-12)
            assert err < 1e-6, (causal, which, err)


def test_element_mask_expands_blocks_and_applies_causal():
    m = np.array([[1, 0], [1, 1]], bool)
    e = element_mask(m, 3, 2, causal=True)
    want = np.array([[1, 0, 0],
                     [1, 1, 0],
                     [1, 1, 1]], bool)
    np.testing.assert_array_equal(e, want)
    e = element_mask(m, 3, 2, causal=False)
    want = np.array([[1, 1, 0],
                     [1, 1, 0],
                     [1, 1, 1]], bool)
    np.testing.assert_array_equal(e, want)
