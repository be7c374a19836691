"""Exact IO-aware attention for B200 (sm_100a): forward and backward.

The compute lives in ``libfa_sm100.so`` (hand-written CUDA, C ABI in
``include/fa.h``).  This package only marshals arguments to it; PyTorch is
used for device memory and streams.

Low-level entry points (same names as the C ABI): ``fa_forward``,
``fa_forward_ex``, ``fa_backward``, ``fa_backward_ex``,
``fa_backward_noalloc``, ``fa_forward_blocksparse``, ``fa_backward_blocksparse``,
``fa_forward_splitkv``, ``fa_splitkv_default_splits``, ``fa_splitkv_workspace_size``,
``fa_backward_workspace_size``, ``fa_forward_fp8``, ``fa_quantize_fp8``,
``fa_set_forward_key_tile``, ``fa_forward_key_tile``,
``fa_status_string``, ``fa_device_status``, ``fa_set_wait_timeout_ns``,
``fa_selftest_wait_timeout``.

Convenience wrappers that allocate outputs with torch:
``attention_forward(q, k, v, scale=None, causal=False, block_mask=None)
-> (o, lse)`` and ``attention_backward(q, k, v, o, do, lse, scale=None,
causal=False, block_mask=None) -> (dq, dk, dv)``, and
``attention_decode(q, k, v, scale=None, causal=False, num_splits=None)
-> (o, lse)`` for N_q queries against N_k keys (split-KV), and the FP8
forward ``attention_forward_fp8(q8, k8, v8, q_descale, k_descale, v_descale,
scale=None, causal=False) -> (o, lse)`` with ``quantize_fp8(x) -> (codes,
descale)`` for its E4M3 inputs.

The shared library is loaded on first use of any of these names (so the
``build`` submodule can run before it exists); using them without the built
library raises ImportError -- there is no fallback.
"""
_NATIVE = {
    "EXPORTS", "FA_BF16", "FA_FP32", "FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED",
    "FA_ERR_MISALIGNED", "FA_ERR_WORKSPACE", "FA_ERR_CUDA", "FA_ERR_DEVICE_TIMEOUT",
    "FA_NOALLOC_SCRATCH_BYTES", "FaError", "LIB_PATH", "library", "fa_forward",
    "fa_forward_ex", "fa_backward", "fa_backward_ex", "fa_backward_noalloc",
    "fa_backward_workspace_size", "fa_status_string", "fa_device_status",
    "fa_set_wait_timeout_ns", "fa_selftest_wait_timeout", "fa_forward_blocksparse",
    "fa_backward_blocksparse", "fa_forward_splitkv", "fa_splitkv_default_splits",
    "fa_splitkv_workspace_size", "fa_forward_fp8", "fa_quantize_fp8",
    "fa_set_forward_key_tile", "fa_forward_key_tile",
}
_API = {"attention_forward", "attention_backward", "attention_decode",
        "attention_forward_fp8", "quantize_fp8"}


def __getattr__(name):
    if name in _NATIVE:
        from . import _native
        return getattr(_native, name)
    if name in _API:
        from . import api
        return getattr(api, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(set(globals()) | _NATIVE | _API)
