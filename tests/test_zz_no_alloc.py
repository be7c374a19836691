"""The allocation-free backward, fa_backward_noalloc.

Some callers cannot allocate device memory or hand the library a workspace:
their device memory belongs to an allocator they cannot reach, they run as a
plugin or callback that only receives tensors, or they must never call
cudaMalloc (which can synchronise the whole device).  For them the library
offers fa_backward_noalloc, which takes its scratch from a fixed array built
into the library.  These tests call it through the C ABI and check that it
gives the same gradients as fa_backward, on two calls in a row, so the second
call must not be disturbed by what the first one left in the shared array.
Both entry points run the same kernels, which accumulate every gradient in a
fixed order (no atomics), so the gradients must agree bit for bit; the
parity tests' tolerance would hide a scratch-reuse mistake.
"""
import math

import pytest
import torch

import workloads


def _compare(B, H, N, d, causal, seed):
    import exact_io_aware_99_b200 as fa
    scale = 1.0 / math.sqrt(d)
    x = workloads.random_case(B, H, N, d, seed)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    ref = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=causal)
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    fa.fa_backward_noalloc(q, k, v, o, do, lse, got[0], got[1], got[2], B, H, N, d, scale,
                           causal)
    torch.cuda.synchronize()
    st, site = fa.fa_device_status(reset=True)
    assert st == fa.FA_OK, f"device wait timed out at site {site:#x}"
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert torch.isfinite(g.float()).all(), name
        assert torch.equal(g, r), (
            f"{name}: differs from fa_backward, max abs diff "
            f"{float((g.float() - r.float()).abs().max()):.3g}")


@pytest.mark.gpu
def test_noalloc_backward_matches_fa_backward_on_two_calls_in_a_row():
    # First call: also performs the one-time lookup of the array's address.
    _compare(1, 2, 300, 128, True, 11)
    # Second call, other shape and inputs: the array still holds the first
    # call's values and must be re-initialised by this call.
    _compare(2, 3, 700, 64, False, 12)


def test_noalloc_backward_rejects_problems_larger_than_its_scratch():
    # Rejected on the host before any device work (fake, aligned pointers).
    import exact_io_aware_99_b200 as fa
    A = 1 << 20
    B, H, N, d = 64, 64, 4096, 128
    assert fa.fa_backward_workspace_size(B, H, N, d) > fa.FA_NOALLOC_SCRATCH_BYTES
    st = fa.fa_backward_noalloc(A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 7 * A, 8 * A, 9 * A,
                                B, H, N, d, 0.1, 1, stream=0, check=False)
    assert st == fa.FA_ERR_WORKSPACE
