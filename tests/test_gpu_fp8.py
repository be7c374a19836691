"""GPU parity for the FP8 forward (fa_forward_fp8) and the per-tensor E4M3
quantiser (fa_quantize_fp8).

The FP8 forward rounds the probabilities to E4M3 before P V, which the
oracle (exact attention of the dequantised inputs) does not do, so:

* on inputs whose probabilities are exact E4M3 values
  (``workloads.fp8_exact_case``) the kernel must match the oracle up to the
  bf16 rounding of O (half an ulp, at most 2^-8 |O|), the row sum's share
  of the FMA-pipe 2^x error (1.2e-4 |O|) and the tensor core's
  accumulation, (2^-20 + (ceil(N/32) + 2) 2^-24) max|V|, derived from the
  MMA's accumulation window, which a test below measures;
* on iid-normal inputs it must stay within ``oracle.fp8.p_rounding_bound``
  (the most rounding P to E4M3 can move each element) plus the same
  allowance and 1.2e-4 max|V| for the 2^x error on the rounded P;
* LSE, computed from the unrounded fp32 probabilities, must agree to 1e-3.

The quantiser must reproduce the seeded generator's per-tensor quantisation
(one fp32 quotient, one fp32 product, round to nearest even) bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from gpu_cases import TOL_LSE, l2_group_heads, np64
from oracle.fp8 import dequantize, forward, p_rounding_bound

pytestmark = pytest.mark.gpu


def fa():
    import exact_io_aware_99_b200 as m
    return m


def run_fp8(x, scale, causal):
    """Run fa_forward_fp8 on the case's codes, descales passed as device
    scalars; returns O and LSE on the GPU."""
    m = fa()
    q8, k8, v8 = (x[n].cuda() for n in ("q8", "k8", "v8"))
    ds = {n: torch.tensor([x[n + "_descale"]], device="cuda", dtype=torch.float32)
          for n in ("q", "k", "v")}
    o, lse = m.attention_forward_fp8(q8, k8, v8, ds["q"], ds["k"], ds["v"], scale, causal)
    torch.cuda.synchronize()
    st, site = m.fa_device_status(reset=True)
    assert st == 0, f"device wait timed out at site {site:#x}"
    return o, lse


# Accumulation window of the E4M3 x E4M3 -> fp32 MMA, measured on B200 by
# test_mma_window_keeps_25_binades_below_the_group_max: inside one 32-key
# k-step, products down to 2^-25 of the step's largest are summed exactly and
# smaller ones are dropped.  With each step's sum then added to the fp32
# accumulator (2^-24 relative per add), the error of sum_j P_j V_jc is at most
#   sum_steps (32 2^-25 M_step + 2^-24 |partial sum|)
# where M_step <= max_j in step P_j max|V| and |partial sum| <= l max|V|; the
# steps' largest P add up to at most l = sum_j P_j, so after the division by l
# (one more fp32 rounding) |err(O)| <= (2^-20 + (n_steps + 2) 2^-24) max|V|.
WINDOW_BINADES = 25


def accumulation_bound(n_keys):
    """Most the P V accumulation can move an element of O, per max|V|."""
    n_steps = -(-max(n_keys, 1) // 32)
    return 32 * 2.0 ** -WINDOW_BINADES + (n_steps + 2) * 2.0 ** -24


def half_ulp_bf16(x):
    """Half the spacing of the bf16 grid at |x| (8 significant bits): the most
    rounding to bf16 can move a value of that magnitude."""
    a = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(a)) - 8.0)


# Relative error of the FMA-pipe 2^x that takes part of the exponentials
# (its fp32 steps are pinned below 1.2e-4 in test_exp2_poly.py).
EXP2_FMA_REL = 1.2e-4


def allowance(ro, go, vmax, n_keys):
    """Rounding O to bf16 (half an ulp at the larger of the reference and
    the result, so a result that crossed a power of two is covered) plus the
    tensor core's accumulation of the E4M3 products of P V (derived above
    from the measured window).  Returns (rounding part, accumulation part)."""
    big = np.maximum(np.abs(ro), np.abs(go))
    # the fp32 normalisation by 1/l (a reciprocal and a product) adds a few
    # fp32 ulps of |O| before the bf16 rounding; the row sum l takes the
    # fp32 probabilities, some from the FMA-pipe 2^x, which moves l, hence
    # O, by at most EXP2_FMA_REL of |O| (P itself lands on the same E4M3
    # value: its error is far below half an E4M3 step)
    return (half_ulp_bf16(big) + (2.0 ** -22 + EXP2_FMA_REL) * big,
            accumulation_bound(n_keys) * vmax)


def compare(x, o, lse, scale, causal, heads=None, exact=False):
    B, H = x["q8"].shape[:2]
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    worst = 0.0
    worst_acc = 0.0  # share of the accumulation term used beyond rounding
    for b, h in pairs:
        q = dequantize(x["q8"][b, h], x["q_descale"])
        k = dequantize(x["k8"][b, h], x["k_descale"])
        v = dequantize(x["v8"][b, h], x["v_descale"])
        ro, rl = forward(x["q8"][b, h], x["k8"][b, h], x["v8"][b, h], x["q_descale"],
                         x["k_descale"], x["v_descale"], scale, causal)
        go, gl = np64(o[b, h]), np64(lse[b, h])
        assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
        rnd, acc = allowance(ro, go, float(np.abs(v).max()), ro.shape[0])
        if not exact:
            # rounding P to E4M3, plus the FMA-pipe 2^x's relative error on the
            # probabilities that are rounded (sum P = 1 after normalisation)
            rnd = (rnd + p_rounding_bound(q, k, v, scale, causal)
                   + EXP2_FMA_REL * float(np.abs(v).max()))
        tol = rnd + acc
        err = np.abs(go - ro)
        bad = err > tol
        assert not bad.any(), (f"head ({b},{h}): {int(bad.sum())} elements outside the bound, "
                               f"worst excess {float((err - tol).max()):.3g}")
        worst = max(worst, float((err / tol).max()))
        worst_acc = max(worst_acc, float((np.maximum(err - rnd, 0.0) / acc).max()))
        el = float(np.max(np.abs(gl - rl)))
        assert el <= TOL_LSE, f"LSE max abs err {el:.3g}"
    print(f"worst |err| / allowed = {worst:.3g}; accumulation term used {worst_acc:.3g}")
    return worst


@pytest.mark.parametrize("d", [64, 80, 128])
@pytest.mark.parametrize("N,causal", [(128, False), (300, True), (1000, False), (129, True)])
def test_exact_probabilities_match_tightly(N, d, causal):
    x = workloads.fp8_exact_case(1, 2, N, d, 2000 + N + d)
    o, lse = run_fp8(x, math.log(2.0), causal)
    compare(x, o, lse, math.log(2.0), causal, exact=True)


@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 2, 300, 128, True),
    (2, 1, 257, 64, False),
    (1, 3, 129, 80, True),
    (1, 1, 1, 128, False),
    (1, 1, 1, 64, True),
    (1, 2, 1024, 128, True),
    (2, 2, 640, 128, False),
])
def test_random_inputs_within_the_rounding_bound(B, H, N, d, causal):
    x = workloads.fp8_random_case(B, H, N, d, 2100 + N + d)
    o, lse = run_fp8(x, 1 / math.sqrt(d), causal)
    compare(x, o, lse, 1 / math.sqrt(d), causal)


@pytest.mark.parametrize("causal", [False, True])
def test_growing_scores_force_rescales(causal):
    # keys grow along the sequence, so the row max keeps rising past the
    # lazy threshold and O is rescaled in tensor memory many times
    N, d = 900, 128
    g = torch.Generator().manual_seed(2200)
    q = torch.randn(1, 1, N, d, generator=g).abs() + 0.5
    k = (torch.randn(1, 1, N, d, generator=g).abs() + 0.5) * torch.linspace(0.1, 3.0, N)[:, None]
    v = torch.randn(1, 1, N, d, generator=g)
    x = {}
    for name, t in (("q", q), ("k", k), ("v", v)):
        x[name + "8"], x[name + "_descale"] = workloads.quantize_e4m3(t)
    o, lse = run_fp8(x, 1 / math.sqrt(d), causal)
    compare(x, o, lse, 1 / math.sqrt(d), causal)


def test_no_descale_pointers_mean_one():
    # E4M3 roundings of N(0, 1) values, for which 1 is the natural factor
    m = fa()
    g = torch.Generator().manual_seed(2300)
    x = {n + "8": torch.randn(1, 1, 200, 64, generator=g).to(torch.float8_e4m3fn)
         .view(torch.uint8).contiguous() for n in ("q", "k", "v")}
    q8, k8, v8 = (x[n].cuda() for n in ("q8", "k8", "v8"))
    o, lse = m.attention_forward_fp8(q8, k8, v8, None, None, None, 0.125, False)
    torch.cuda.synchronize()
    y = dict(x, q_descale=1.0, k_descale=1.0, v_descale=1.0)
    compare(y, o, lse, 0.125, False)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n", [1, 7, 1000, 12345, (1 << 20) + 3])
def test_quantiser_matches_the_generator_bit_for_bit(dtype, n):
    m = fa()
    g = torch.Generator().manual_seed(2400 + n)
    x = (torch.randn(n, generator=g) * 3.0).to(dtype)
    codes, ds = m.quantize_fp8(x.cuda())
    torch.cuda.synchronize()
    ref_codes, ref_ds = workloads.quantize_e4m3(x.float())
    assert np.float32(ds.item()) == np.float32(ref_ds)
    assert torch.equal(codes.cpu(), ref_codes)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantiser_tiny_amax_matches_the_generator(dtype):
    # amax ~1e-37: 448 / amax overflows fp32, so the factor and the descale
    # are 1 and the codes are signed zeros (no NaN codes from 0 * inf)
    m = fa()
    x = torch.tensor([0.0, 1e-37, -3e-37, 0.0, 5e-38, -0.0] * 5, dtype=torch.float32).to(dtype)
    codes, ds = m.quantize_fp8(x.cuda())
    torch.cuda.synchronize()
    ref_codes, ref_ds = workloads.quantize_e4m3(x.float())
    assert ds.item() == 1.0 and ref_ds == 1.0
    assert torch.equal(codes.cpu(), ref_codes)


def test_quantiser_all_zero_input():
    m = fa()
    codes, ds = m.quantize_fp8(torch.zeros(333, device="cuda", dtype=torch.bfloat16))
    torch.cuda.synchronize()
    assert ds.item() == 1.0 and not codes.any()


def test_quantise_then_forward_reads_descales_on_the_device():
    m = fa()
    B, H, N, d = 1, 2, 384, 128
    g = torch.Generator().manual_seed(2500)
    xs = {n: (torch.randn(B, H, N, d, generator=g) * s).to(torch.bfloat16)
          for n, s in (("q", 2.0), ("k", 0.5), ("v", 4.0))}
    qc, qd = m.quantize_fp8(xs["q"].cuda())
    kc, kd = m.quantize_fp8(xs["k"].cuda())
    vc, vd = m.quantize_fp8(xs["v"].cuda())
    o, lse = m.attention_forward_fp8(qc, kc, vc, qd, kd, vd, None, True)
    torch.cuda.synchronize()
    x = {"q8": qc.cpu(), "k8": kc.cpu(), "v8": vc.cpu(), "q_descale": qd.item(),
         "k_descale": kd.item(), "v_descale": vd.item()}
    compare(x, o, lse, 1 / math.sqrt(d), True)


def test_full_size_workload_group_heads():
    # the benchmark's FP8 workload in its own launch configuration; the first
    # head of every L2 head group (E4M3 K and V: one byte per element) and
    # every head of the last group compared with the oracle
    w = workloads.WORKLOADS["fp8_causal_d128"]
    x = workloads.make_fp8_inputs(w)
    o, lse = run_fp8(x, w.scale, w.causal)
    compare(x, o, lse, w.scale, w.causal,
            heads=l2_group_heads(w.B, w.H, w.N, w.d, w.causal, kv_bytes=1))


def test_bad_arguments_are_rejected():
    m = fa()
    q = torch.zeros(1, 1, 128, 96, device="cuda", dtype=torch.uint8)
    o = torch.empty(1, 1, 128, 96, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(1, 1, 128, device="cuda", dtype=torch.float32)
    st = m.fa_forward_fp8(q, q, q, None, None, None, o, lse, 1, 1, 128, 96, 0.1, 0, check=False)
    assert st == m.FA_ERR_UNSUPPORTED              # d = 96
    q = torch.zeros(1, 1, 128, 64, device="cuda", dtype=torch.uint8)
    o = torch.empty(1, 1, 128, 64, device="cuda", dtype=torch.bfloat16)
    st = m.fa_forward_fp8(q.data_ptr() + 1, q, q, None, None, None, o, lse, 1, 1, 127, 64, 0.1,
                          0, check=False)
    assert st == m.FA_ERR_MISALIGNED
    st = m.fa_forward_fp8(None, q, q, None, None, None, o, lse, 1, 1, 128, 64, 0.1, 0,
                          check=False)
    assert st == m.FA_ERR_INVALID_ARG
    st = m.fa_forward_fp8(q, q, q, None, None, None, o, lse, 1, 1, 128, 64, float("nan"), 0,
                          check=False)
    assert st == m.FA_ERR_INVALID_ARG
    ds = torch.empty(1, device="cuda", dtype=torch.float32)
    assert m.fa_quantize_fp8(o, m.FA_BF16, 0, q, ds, check=False) == m.FA_ERR_INVALID_ARG
    assert m.fa_quantize_fp8(o, 7, 10, q, ds, check=False) == m.FA_ERR_UNSUPPORTED


def test_mma_window_keeps_25_binades_below_the_group_max():
    # The premise of accumulation_bound.  Scale ln 2 makes each score its
    # base-2 exponent.  Key tile 0 (keys 0-127) scores 0, so the reference max
    # is 0; in key tile 1 keys 128 and 129 score 8 (no rescale: growth 8 is
    # not above the threshold), P = 2^8, with V = +256 and -256: products of
    # +-2^16 that cancel exactly, in the 32-key step 128..159.  Every other key
    # of tile 1 scores -8 (P = 2^-8) with V = 2^-9, 2^-8, ...: small products
    # 2^-17 .. 2^-2 sharing that step.  Those at least 2^-25 of 2^16 (2^-9 and
    # up) must survive; O is exact attention up to bf16 rounding.
    m = fa()
    N, d = 256, 64
    q = torch.zeros(1, 1, N, d)
    q[..., 0] = 1.0
    k = torch.zeros(1, 1, N, d)
    k[0, 0, 128:, 0] = -8.0
    k[0, 0, 128:130, 0] = 8.0
    v = torch.zeros(1, 1, N, d)
    for c in range(16):
        v[0, 0, 128:, c] = 2.0 ** (-9 + c)
    v[0, 0, 128, :] = 256.0
    v[0, 0, 129, :] = -256.0

    def codes(x):
        return x.to(torch.float8_e4m3fn).view(torch.uint8).contiguous().cuda()

    o, _ = m.attention_forward_fp8(codes(q), codes(k), codes(v), None, None, None,
                                   math.log(2.0), False)
    torch.cuda.synchronize()
    l = 128 + 2 * 256 + 126 * 2.0 ** -8
    got = o[0, 0, 0].float().cpu().numpy()
    for c in range(16):
        small = 2.0 ** (-8 - 9 + c)          # one small product
        if 16 - (-17 + c) > WINDOW_BINADES:  # outside the window: not asserted
            continue
        exact = 126 * small / l
        assert abs(got[c] - exact) <= 2.0 ** -8 * exact, (c, got[c], exact)

