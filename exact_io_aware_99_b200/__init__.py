"""Exact IO-aware attention for B200 (sm_100a): forward and backward.

The compute lives in ``libfa_sm100.so`` (hand-written CUDA, C ABI in
``include/fa.h``).  This package only marshals arguments to it; PyTorch is
used for device memory and streams.

Low-level entry points (same names as the C ABI): ``fa_forward``,
``fa_forward_ex``, ``fa_backward``, ``fa_backward_ex``,
``fa_backward_workspace_size``, ``fa_status_string``, ``fa_device_status``,
``fa_set_wait_timeout_ns``, ``fa_selftest_wait_timeout``.

Convenience wrappers that allocate outputs with torch:
``attention_forward(q, k, v, scale=None, causal=False) -> (o, lse)`` and
``attention_backward(q, k, v, o, do, lse, scale=None, causal=False)
-> (dq, dk, dv)``.
"""
from ._native import (EXPORTS, FA_BF16, FA_ERR_CUDA, FA_ERR_DEVICE_TIMEOUT,  # noqa: F401
                      FA_ERR_INVALID_ARG, FA_ERR_MISALIGNED, FA_ERR_UNSUPPORTED,
                      FA_ERR_WORKSPACE, FA_FP32, FA_OK, FaError, LIB_PATH,
                      fa_backward, fa_backward_ex, fa_backward_workspace_size,
                      fa_device_status, fa_forward, fa_forward_ex, fa_selftest_wait_timeout,
                      fa_set_wait_timeout_ns, fa_status_string, library)
from .api import attention_backward, attention_forward  # noqa: F401
