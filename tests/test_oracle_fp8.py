"""Pins for the FP8 oracle (oracle/fp8.py), CPU only.

* E4M3 decoding against torch's float8_e4m3fn conversion (a library routine)
  for all 256 codes, and against values the format fixes by hand.
* ``forward`` against identities of the definition: the descale factors of Q
  and K multiply the scores like the attention scale, V's descale multiplies
  O and leaves LSE alone, and identical keys give the mean of the visible V
  rows.
* ``p_rounding_bound`` against the rounding itself: probabilities taken
  against arbitrary reference maxima (per key block, as an online softmax
  does), rounded to E4M3 by torch, divided by the unrounded sum, never move O
  further than the bound.
* The exact case of ``workloads.fp8_exact_case``: every such probability is
  an E4M3 value, so that rounding changes nothing.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention_forward
from oracle.fp8 import (E4M3_MAX, dequantize, e4m3_decode, forward,
                        p_rounding_bound)

RNG = np.random.default_rng(8008)


def rn_e4m3(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even to E4M3 through torch (values <= 448 here)."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def test_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    np.testing.assert_array_equal(ours[~nan], ref[~nan].astype(np.float64))
    # signed zero
    assert np.signbit(ours[0x80]) and ours[0x80] == 0.0


@pytest.mark.parametrize("code,value", [
    (0x7E, 448.0),            # 0 1111 110: 1.75 * 2^8, the largest finite value
    (0x38, 1.0),              # exponent field 7 = bias
    (0xB8, -1.0),
    (0x08, 2.0 ** -6),        # smallest normal
    (0x07, 7 * 2.0 ** -9),    # largest subnormal
    (0x01, 2.0 ** -9),        # smallest subnormal
    (0x0F, 1.875 * 2.0 ** -6),
    (0x78, 256.0),
    (0x00, 0.0),
])
def test_decode_values_fixed_by_the_format(code, value):
    assert e4m3_decode(np.array([code], dtype=np.uint8))[0] == value
    assert E4M3_MAX == 448.0


def codes(shape):
    x = RNG.standard_normal(shape).astype(np.float32)
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_qk_descales_act_like_the_attention_scale(causal):
    q8, k8, v8 = codes((2, 33, 8)), codes((2, 33, 8)), codes((2, 33, 8))
    o1, l1 = forward(q8, k8, v8, 0.75, 0.5, 1.0, 0.3, causal)
    o2, l2 = forward(q8, k8, v8, 1.0, 1.0, 1.0, 0.3 * 0.75 * 0.5, causal)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_v_descale_scales_o_only():
    q8, k8, v8 = codes((3, 20, 8)), codes((3, 20, 8)), codes((3, 20, 4))
    o1, l1 = forward(q8, k8, v8, 0.1, 0.2, 1.0, 0.5)
    o2, l2 = forward(q8, k8, v8, 0.1, 0.2, 0.125, 0.5)
    np.testing.assert_allclose(o2, 0.125 * o1, atol=1e-14)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_the_mean_of_visible_values(causal):
    n = 17
    k8 = np.tile(codes((1, 1, 6)), (1, n, 1))
    q8, v8 = codes((1, n, 6)), codes((1, n, 5))
    o, lse = forward(q8, k8, v8, 0.5, 0.25, 2.0, 0.4, causal)
    v = dequantize(v8, 2.0)[0]
    s = 0.4 * dequantize(q8, 0.5)[0] @ dequantize(k8[:, :1], 0.25)[0, 0]
    for i in range(n):
        cnt = i + 1 if causal else n
        np.testing.assert_allclose(o[0, i], v[:cnt].mean(axis=0), atol=1e-12)
        np.testing.assert_allclose(lse[0, i], s[i] + math.log(cnt), atol=1e-12)


def rounded_online(q, k, v, scale, causal, block, ref_gap):
    """O with probabilities rounded to E4M3, each key block's probabilities
    taken against its own reference maximum (the row's running max of the
    blocks so far, lowered by ref_gap[t] in log2 units, at most 8), the
    output summed in fp64 and divided by the unrounded sum."""
    n = q.shape[0]
    s = scale * (q @ k.T)
    if causal:
        s = np.where(np.arange(n)[None, :] > np.arange(n)[:, None], -np.inf, s)
    num = np.zeros((n, v.shape[1]))
    den = np.zeros(n)
    m_run = np.full(n, -np.inf)
    ref = np.full(n, -np.inf)
    for t, j0 in enumerate(range(0, n, block)):
        sb = s[:, j0:j0 + block]
        m_run = np.maximum(m_run, sb.max(axis=1))
        new_ref = m_run - ref_gap[t] * math.log(2.0)
        ok = np.isfinite(new_ref)
        # rescale what was accumulated against the old reference
        f = np.where(np.isfinite(ref) & ok, np.exp(ref - new_ref), 1.0)
        num *= f[:, None]
        den *= f
        ref = np.where(ok, new_ref, ref)
        p = np.where(np.isfinite(sb), np.exp(sb - ref[:, None]), 0.0)
        assert p.max() <= 256.0 + 1e-9
        num += rn_e4m3(p) @ v[j0:j0 + block]
        den += p.sum(axis=1)
    return num / den[:, None]


@pytest.mark.parametrize("spread", [0.5, 3.0, 12.0])
@pytest.mark.parametrize("causal", [False, True])
def test_rounding_stays_within_the_bound(spread, causal):
    n, d = 48, 8
    for trial in range(4):
        q = RNG.standard_normal((n, d)) * spread
        k = RNG.standard_normal((n, d))
        v = RNG.standard_normal((n, 5)) * 3.0
        scale = 1 / math.sqrt(d)
        o, _ = attention_forward(q, k, v, scale, causal)
        bound = p_rounding_bound(q, k, v, scale, causal)
        gaps = RNG.uniform(0.0, 8.0, size=(n + 15) // 16)
        if trial == 0:
            gaps[:] = 0.0
        got = rounded_online(q, k, v, scale, causal, 16, gaps)
        err = np.abs(got - o)
        assert np.all(err <= bound * (1 + 1e-9) + 1e-13), float((err - bound).max())
        # and the bound is not vacuous: it stays below the full rounding size
        assert np.all(bound <= 2.0 ** -4 * (np.abs(v).max() + 1e-300) + n * 2.0 ** -10 * 3.0 * 5)


def test_bound_is_tight_enough_to_see_a_dropped_probability():
    # dropping the largest probability of a row moves O far outside the bound
    n, d = 32, 8
    q = RNG.standard_normal((n, d))
    k = RNG.standard_normal((n, d))
    v = RNG.standard_normal((n, 4))
    s = 0.4 * (q @ k.T)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    o, _ = attention_forward(q, k, v, 0.4)
    jmax = np.argmax(s, axis=1)
    p_bad = p.copy()
    p_bad[np.arange(n), jmax] = 0.0
    o_bad = (p_bad @ v) / p.sum(axis=1, keepdims=True)
    bound = p_rounding_bound(q, k, v, 0.4)
    assert np.any(np.abs(o_bad - o) > bound)


@pytest.mark.parametrize("causal", [False, True])
def test_exact_case_probabilities_are_e4m3_values(causal):
    x = workloads.fp8_exact_case(1, 2, 70, 32, 5)
    q = dequantize(x["q8"], x["q_descale"])
    k = dequantize(x["k8"], x["k_descale"])
    v = dequantize(x["v8"], x["v_descale"])
    for h in range(2):
        x2 = (q[0, h] @ k[0, h].T)            # scores / ln 2 = base-2 units
        assert np.all(x2 == np.round(x2)) and np.abs(x2).max() <= 4
        # every reference max in the row's range keeps 2^(x - m) exact
        o, _ = attention_forward(q[0, h], k[0, h], v[0, h], math.log(2.0), causal)
        for gaps in ([0.0] * 5, [3.0, 8.0, 0.0, 5.0, 1.0]):
            got = rounded_online(q[0, h], k[0, h], v[0, h], math.log(2.0), causal, 16,
                                 np.array(gaps))
            np.testing.assert_allclose(got, o, atol=1e-12, rtol=0)


def test_quantize_generator_maps_amax_to_448():
    x = torch.randn(3, 1000) * 7.0
    c, ds = workloads.quantize_e4m3(x)
    vals = e4m3_decode(c.numpy())
    assert np.float32(ds) == np.float32(x.abs().max()) / np.float32(448.0)
    assert np.abs(vals).max() == 448.0
    rel = np.abs(vals * ds - x.numpy()) / np.maximum(np.abs(x.numpy()), 2.0 ** -6 * ds)
    assert rel.max() <= 2.0 ** -4 + 1e-6
    c0, ds0 = workloads.quantize_e4m3(torch.zeros(5))
    assert ds0 == 1.0 and not c0.any()


def test_quantize_generator_tiny_amax_takes_the_tensor_as_it_is():
    # 448 / amax overflows fp32 for amax below ~1.3e-36: no factor maps amax
    # to 448, so the factor and the descale are both 1 and every value
    # (|x| < 2^-10) rounds to a signed zero -- never to a NaN code.
    x = torch.tensor([0.0, 1e-37, -3e-37, 0.0, 5e-38, -0.0], dtype=torch.float32)
    with np.errstate(over="ignore"):
        assert not math.isfinite(np.float32(448.0) / np.float32(x.abs().max()))
    c, ds = workloads.quantize_e4m3(x)
    assert ds == 1.0
    assert set(c.tolist()) <= {0x00, 0x80}
    assert np.all(e4m3_decode(c.numpy()) == 0.0)
    # just above the overflow point the ordinary rule applies
    y = torch.tensor([0.0, 2e-36, -1e-36], dtype=torch.float32)
    c1, ds1 = workloads.quantize_e4m3(y)
    assert np.float32(ds1) == np.float32(2e-36) / np.float32(448.0)
    assert np.abs(e4m3_decode(c1.numpy())).max() == 448.0
