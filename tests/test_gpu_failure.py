"""Failure detection without a GPU fault: a device-side wait on a barrier that
nothing completes must give up after its time limit, record its site in the
status word, and let the kernel return; the context stays usable."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    import exact_io_aware_99_b200 as fa
    fa.fa_device_status(reset=True)
    fa.fa_set_wait_timeout_ns(50_000_000)  # 50 ms
    try:
        fa.fa_selftest_wait_timeout()
        st, site = fa.fa_device_status(reset=True)
    finally:
        fa.fa_set_wait_timeout_ns(0)
    assert st == fa.FA_ERR_DEVICE_TIMEOUT
    assert site == 0x7E57
    # the status word was reset and the context still works
    st, site = fa.fa_device_status(reset=True)
    assert st == fa.FA_OK and site == 0
    x = workloads.random_case(1, 1, 64, 64, 1, grad=False)
    o, lse = fa.attention_forward(x["q"].cuda(), x["k"].cuda(), x["v"].cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert fa.fa_device_status(reset=True)[0] == fa.FA_OK
