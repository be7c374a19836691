"""GPU backward parity: dQ, dK, dV from the C ABI against the fp64 oracle's
analytic backward on the same seeded inputs (the GPU's own forward supplies O
and LSE, as in training)."""
import math

import pytest
import torch

import workloads
from gpu_cases import check_backward, l2_group_heads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,d,causal", [(1, 32, False), (40, 64, True), (129, 80, False),
                                        (150, 128, True)])
def test_fp32_backward(N, d, causal):
    x = workloads.random_case(1, 2, N, d, 300 + N, dtype=torch.float32)
    w = check_backward(x["q"], x["k"], x["v"], x["do"], 1 / math.sqrt(d), causal)
    # fp32 arithmetic throughout: far inside the bf16 tolerance (the errors
    # are relative to max(max|ref|, 1e-4), so the all-zero dQ/dK at N = 1
    # read as abs error / 1e-4)
    assert max(w.values()) < 5e-3


@pytest.mark.parametrize("d", [64, 80, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 128, 129, 300, 1000])
def test_bf16_backward_small_shapes(N, d, causal):
    x = workloads.random_case(1, 2, N, d, 500 + 3 * d + N + causal)
    check_backward(x["q"], x["k"], x["v"], x["do"], 1 / math.sqrt(d), causal)


def test_bf16_backward_several_heads():
    x = workloads.random_case(2, 3, 700, 128, 4242)
    check_backward(x["q"], x["k"], x["v"], x["do"], 1 / math.sqrt(128), True)


def test_bf16_backward_is_bitwise_reproducible():
    # Every gradient tile is accumulated by one CTA in a fixed order (no
    # atomics), whichever CTA ends up running it: two runs agree bit for bit.
    from gpu_cases import gpu_backward, gpu_forward
    x = workloads.random_case(1, 4, 1024, 64, 7)
    o, lse = gpu_forward(x["q"], x["k"], x["v"], 0.125, True)
    a = gpu_backward(x["q"], x["k"], x["v"], o, x["do"], lse, 0.125, True)
    b = gpu_backward(x["q"], x["k"], x["v"], o, x["do"], lse, 0.125, True)
    for ga, gb in zip(a, b):
        assert torch.equal(ga, gb)


# Full-size workloads in the benchmark's launch configuration: the first
# head of every L2 head group and every head of the last group (see
# gpu_cases.l2_group_heads) are checked completely.
@pytest.mark.parametrize("name", ["causal_d128", "long_d128", "gpt3_d80"])
def test_full_size_workload_backward(name):
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w)
    check_backward(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal,
                   heads=l2_group_heads(w.B, w.H, w.N, w.d, w.causal))


def test_gradients_at_16_byte_aligned_addresses_match_the_32_byte_path():
    # The gradient rows are written with 32-byte stores when dQ, dK and dV are
    # 32-byte aligned and with 16-byte stores otherwise: both give the same bits.
    import exact_io_aware_99_b200 as fa
    from gpu_cases import gpu_forward
    B, H, N, d = 1, 3, 300, 128
    x = workloads.random_case(B, H, N, d, 4343)
    o, lse = gpu_forward(x["q"], x["k"], x["v"], 1 / math.sqrt(d), True)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    n = B * H * N * d
    wb = fa.fa_backward_workspace_size(B, H, N, d)
    ws = torch.empty(wb, device="cuda", dtype=torch.uint8)
    outs = []
    for off in (0, 8):  # elements: 8 bf16 = 16 bytes
        bufs = [torch.empty(n + 16, device="cuda", dtype=torch.bfloat16) for _ in range(3)]
        g = [b_[off:off + n].view(B, H, N, d) for b_ in bufs]
        assert (g[0].data_ptr() & 31) == (0 if off == 0 else 16)
        fa.fa_backward(q, k, v, o, do, lse, g[0], g[1], g[2], B, H, N, d, 1 / math.sqrt(d),
                       True, ws, wb)
        torch.cuda.synchronize()
        outs.append([t.clone() for t in g])
    st, site = fa.fa_device_status(reset=True)
    assert st == 0, f"device wait timed out at site {site:#x}"
    for a, b in zip(*outs):
        assert torch.equal(a, b)
