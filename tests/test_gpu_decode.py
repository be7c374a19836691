"""GPU parity for the split-KV decode forward (fa_forward_splitkv) against the
fp64 decode oracle on the same seeded inputs: O and LSE, including rows that
see no key, for single queries, ragged query and key counts, several split
counts and the bottom-right causal rule."""
import math

import numpy as np
import pytest
import torch

import workloads
from gpu_cases import TOL_LSE, TOL_O_BF16, np64
from oracle.decode import rect_forward

pytestmark = pytest.mark.gpu


def fa():
    import exact_io_aware_99_b200 as m
    return m


def run_case(B, H, Nq, Nk, d, causal, splits, seed):
    m = fa()
    xq = workloads.random_case(B, H, Nq, d, seed, grad=False)
    xk = workloads.random_case(B, H, Nk, d, seed + 1, grad=False)
    q = xq["q"].cuda()
    k, v = xk["k"].cuda(), xk["v"].cuda()
    o, lse = m.attention_decode(q, k, v, causal=causal, num_splits=splits)
    torch.cuda.synchronize()
    st, site = m.fa_device_status(reset=True)
    assert st == 0, f"device wait timed out at site {site:#x}"
    ro, rl = rect_forward(xq["q"], xk["k"], xk["v"], 1 / math.sqrt(d), causal)
    go, gl = np64(o), np64(lse)
    assert np.all(np.isfinite(go))
    err = float(np.max(np.abs(go - ro)))
    assert err <= TOL_O_BF16, f"O max abs err {err:.3g}"
    np.testing.assert_array_equal(np.isneginf(gl), np.isneginf(rl))
    fin = np.isfinite(rl)
    if fin.any():
        el = float(np.max(np.abs(gl[fin] - rl[fin])))
        assert el <= TOL_LSE, f"LSE max abs err {el:.3g}"
    return rl


@pytest.mark.parametrize("d", [64, 80, 128])
def test_single_query_long_cache(d):
    run_case(2, 3, 1, 1000, d, False, None, 1100 + d)


@pytest.mark.parametrize("splits", [1, 3, 7])
def test_causal_bottom_right_odd_sizes(splits):
    run_case(1, 4, 37, 5000, 64, True, splits, 1200 + splits)


def test_query_tile_pair_ragged():
    # 200 queries = a full query tile and a 72-row second one, 777 keys
    run_case(1, 2, 200, 777, 80, True, 3, 1300)
    run_case(1, 2, 200, 777, 128, False, 4, 1301)


def test_square_problem_matches_dense_definition():
    run_case(1, 2, 300, 300, 128, True, 2, 1400)


def test_more_queries_than_keys_hides_the_first_rows():
    rl = run_case(1, 1, 150, 100, 64, True, 2, 1500)
    assert np.all(np.isneginf(rl[..., :50])) and np.all(np.isfinite(rl[..., 50:]))


def test_more_splits_than_key_tiles_is_clamped():
    m = fa()
    assert m.fa_splitkv_workspace_size(1, 1, 16, 256, 128, 10) == \
        m.fa_splitkv_workspace_size(1, 1, 16, 256, 128, 2)
    run_case(1, 1, 16, 256, 128, False, 10, 1600)


def test_bad_arguments_are_rejected():
    m = fa()
    x = workloads.random_case(1, 1, 128, 64, 1700, grad=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 128), device="cuda", dtype=torch.float32)
    wb = m.fa_splitkv_workspace_size(1, 1, 128, 128, 64, 1)
    ws = torch.empty(wb, device="cuda", dtype=torch.uint8)
    st = m.fa_forward_splitkv(q, k, v, o, lse, 1, 1, 128, 128, 64, 0.125, 0, 0, ws, wb,
                              check=False)
    assert st == m.FA_ERR_INVALID_ARG          # num_splits < 1
    st = m.fa_forward_splitkv(q, k, v, o, lse, 1, 1, 128, 128, 64, 0.125, 0, 1, ws, wb - 256,
                              check=False)
    assert st == m.FA_ERR_WORKSPACE            # workspace too small
