"""Pins for the decode oracle (oracle/decode.py), CPU only: the square case
reduces to the dense oracle, scalar loops agree on rectangular causal
problems, key-chunk partials merge back to the full result, and the
bottom-right causal rule lets the last query see every key."""
import numpy as np
import pytest

from oracle import attention_forward
from oracle.decode import (brute_forward, chunk_forward, merge_partials, rect_forward,
                           visible)

RNG = np.random.default_rng(31337)


def rand(*shape):
    return RNG.standard_normal(shape)


@pytest.mark.parametrize("causal", [False, True])
def test_square_problem_is_the_dense_oracle(causal):
    q, k, v = rand(2, 3, 29, 6), rand(2, 3, 29, 6), rand(2, 3, 29, 6)
    o, lse = rect_forward(q, k, v, 0.4, causal)
    od, ld = attention_forward(q, k, v, 0.4, causal)
    np.testing.assert_allclose(o, od, atol=1e-12)
    np.testing.assert_allclose(lse, ld, atol=1e-12)


@pytest.mark.parametrize("nq,nk", [(1, 9), (3, 10), (5, 5), (6, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_matches_scalar_loops(nq, nk, causal):
    q, k, v = rand(nq, 3), rand(nk, 3), rand(nk, 2)
    o, lse = rect_forward(q, k, v, 0.7, causal)
    ob, lb = brute_forward(q, k, v, 0.7, causal)
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], atol=1e-12)


def test_bottom_right_causal_rule():
    m = visible(3, 7, True)
    # query 0 is position 4 of 7, query 2 the last position
    np.testing.assert_array_equal(m.sum(axis=1), [5, 6, 7])
    assert m[2].all()
    # more queries than keys: the first queries see nothing
    m = visible(5, 3, True)
    np.testing.assert_array_equal(m.sum(axis=1), [0, 0, 1, 2, 3])


@pytest.mark.parametrize("causal", [False, True])
def test_key_chunk_partials_merge_to_the_full_result(causal):
    nq, nk = 7, 50
    q, k, v = rand(2, nq, 5), rand(2, nk, 5), rand(2, nk, 4)
    full_o, full_l = rect_forward(q, k, v, 0.6, causal)
    edges = [0, 13, 14, 30, 50]          # uneven chunks, one of a single key
    parts = [chunk_forward(q, k, v, 0.6, causal, a, b) for a, b in zip(edges, edges[1:])]
    o, lse = merge_partials([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(o, full_o, atol=1e-12)
    np.testing.assert_allclose(lse, full_l, atol=1e-12)


def test_merge_of_hidden_chunks_keeps_zero_and_minus_inf():
    o1 = np.zeros((2, 3))
    l1 = np.array([-np.inf, 0.5])
    o2 = np.ones((2, 3))
    l2 = np.array([-np.inf, -np.inf])
    o, lse = merge_partials([o1, o2], [l1, l2])
    np.testing.assert_array_equal(o[0], 0.0)
    assert np.isneginf(lse[0]) and lse[1] == 0.5
    np.testing.assert_array_equal(o[1], 0.0)


def test_single_query_closed_form():
    k, v = rand(40, 4), rand(40, 3)
    q = rand(1, 4)
    s = 0.9 * (k @ q[0])
    w = np.exp(s - s.max())
    want = (w / w.sum()) @ v
    o, lse = rect_forward(q, k, v, 0.9, False)
    np.testing.assert_allclose(o[0], want, atol=1e-13)
    np.testing.assert_allclose(lse[0], s.max() + np.log(w.sum()), atol=1e-13)
