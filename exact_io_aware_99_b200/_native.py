"""ctypes binding of libfa_sm100.so (the C ABI in include/fa.h).

Argument marshalling only: tensors become device pointers, streams become
cudaStream_t handles, and non-zero status codes become ``FaError``.  Every
step of the computation runs in the library's CUDA kernels; there is no
fallback of any kind, and importing this module fails loudly when the shared
library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_sm100.so")

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_MISALIGNED = -3
FA_ERR_WORKSPACE = -4
FA_ERR_CUDA = -5
FA_ERR_DEVICE_TIMEOUT = -6

FA_BF16 = 0
FA_FP32 = 1

EXPORTS = (
    "fa_forward", "fa_forward_ex", "fa_backward_workspace_size", "fa_backward",
    "fa_backward_ex", "fa_status_string", "fa_last_cuda_error", "fa_device_status",
    "fa_set_wait_timeout_ns", "fa_selftest_wait_timeout", "fa_backward_noalloc",
    "fa_forward_blocksparse", "fa_backward_blocksparse", "fa_forward_splitkv",
    "fa_splitkv_default_splits", "fa_splitkv_workspace_size", "fa_forward_fp8",
    "fa_quantize_fp8", "fa_set_forward_key_tile", "fa_forward_key_tile",
)

# Size of the library's built-in scratch array used by fa_backward_noalloc.
FA_NOALLOC_SCRATCH_BYTES = 64 << 20


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)} ({status})"
        if status == FA_ERR_CUDA:
            msg += f", cuda error {_lib.fa_last_cuda_error()}"
        super().__init__(msg)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m exact_io_aware_99_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_forward.argtypes = [P, P, P, P, P, I, I, I, I, F, I, P]
    lib.fa_forward.restype = I
    lib.fa_forward_ex.argtypes = [P, P, P, P, P, I, I, I, I, F, I, I, P]
    lib.fa_forward_ex.restype = I
    lib.fa_backward_workspace_size.argtypes = [I, I, I, I]
    lib.fa_backward_workspace_size.restype = S
    lib.fa_backward.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P, S, P]
    lib.fa_backward.restype = I
    lib.fa_backward_ex.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P, S, I, P]
    lib.fa_backward_ex.restype = I
    lib.fa_status_string.argtypes = [I]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_cuda_error.argtypes = []
    lib.fa_last_cuda_error.restype = I
    lib.fa_device_status.argtypes = [I, ctypes.POINTER(I)]
    lib.fa_device_status.restype = I
    lib.fa_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
    lib.fa_set_wait_timeout_ns.restype = None
    lib.fa_selftest_wait_timeout.argtypes = [P]
    lib.fa_selftest_wait_timeout.restype = I
    lib.fa_backward_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P]
    lib.fa_forward_blocksparse.argtypes = [P, P, P, P, P, I, I, I, I, F, I, P, I, P]
    lib.fa_forward_blocksparse.restype = I
    lib.fa_backward_blocksparse.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P, I,
                                            P, S, P]
    lib.fa_backward_blocksparse.restype = I
    lib.fa_forward_splitkv.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, I, P, S, P]
    lib.fa_forward_splitkv.restype = I
    lib.fa_splitkv_default_splits.argtypes = [I, I, I, I]
    lib.fa_splitkv_default_splits.restype = I
    lib.fa_splitkv_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.fa_splitkv_workspace_size.restype = S
    lib.fa_backward_noalloc.restype = I
    lib.fa_forward_fp8.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, F, I, P]
    lib.fa_forward_fp8.restype = I
    lib.fa_quantize_fp8.argtypes = [P, I, S, P, P, P]
    lib.fa_quantize_fp8.restype = I
    lib.fa_set_forward_key_tile.argtypes = [I]
    lib.fa_set_forward_key_tile.restype = I
    lib.fa_forward_key_tile.argtypes = [I, I, I]
    lib.fa_forward_key_tile.restype = I
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()  # torch tensor


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream  # torch.cuda.Stream


def _check(st: int, where: str, check: bool) -> int:
    if check and st != FA_OK:
        raise FaError(st, where)
    return st


def status_string(st: int) -> str:
    return _lib.fa_status_string(int(st)).decode()


def fa_forward(q, k, v, o, lse, B, H, N, d, scale, causal, stream=None, check=True) -> int:
    st = _lib.fa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                         float(scale), int(bool(causal)), _stream(stream))
    return _check(st, "fa_forward", check)


def fa_forward_ex(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, stream=None,
                  check=True) -> int:
    st = _lib.fa_forward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                            float(scale), int(bool(causal)), int(dtype), _stream(stream))
    return _check(st, "fa_forward_ex", check)


def fa_backward_workspace_size(B, H, N, d) -> int:
    return int(_lib.fa_backward_workspace_size(B, H, N, d))


def fa_backward(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace,
                workspace_bytes, stream=None, check=True) -> int:
    st = _lib.fa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq),
                          _ptr(dk), _ptr(dv), B, H, N, d, float(scale), int(bool(causal)),
                          _ptr(workspace), int(workspace_bytes), _stream(stream))
    return _check(st, "fa_backward", check)


def fa_backward_ex(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace,
                   workspace_bytes, dtype, stream=None, check=True) -> int:
    st = _lib.fa_backward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                             _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                             int(bool(causal)), _ptr(workspace), int(workspace_bytes),
                             int(dtype), _stream(stream))
    return _check(st, "fa_backward_ex", check)


def fa_status_string(st: int) -> str:
    return status_string(st)


def fa_device_status(reset: bool = True):
    site = ctypes.c_int(0)
    st = _lib.fa_device_status(int(bool(reset)), ctypes.byref(site))
    return st, site.value


def fa_set_wait_timeout_ns(ns: int) -> None:
    _lib.fa_set_wait_timeout_ns(int(ns))


def fa_set_forward_key_tile(keys: int, check=True) -> int:
    """Force the dense bf16 forward's key-tile size (64 or 128) for every
    later call, or restore the built-in table (0)."""
    return _check(_lib.fa_set_forward_key_tile(int(keys)), "fa_set_forward_key_tile", check)


def fa_forward_key_tile(d: int, N: int, causal: bool) -> int:
    """Key-tile size the dense bf16 forward uses for this shape (0: unsupported)."""
    return int(_lib.fa_forward_key_tile(int(d), int(N), int(bool(causal))))


def fa_selftest_wait_timeout(stream=None, check=True) -> int:
    st = _lib.fa_selftest_wait_timeout(_stream(stream))
    return _check(st, "fa_selftest_wait_timeout", check)


def fa_backward_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal,
                        stream=None, check=True) -> int:
    """fa_backward without a workspace argument: the scratch is the
    library's built-in device array (FA_NOALLOC_SCRATCH_BYTES); nothing is
    allocated.  For callers that cannot allocate device memory."""
    st = _lib.fa_backward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                  _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                  int(bool(causal)), _stream(stream))
    return _check(st, "fa_backward_noalloc", check)


def fa_forward_blocksparse(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, mask_heads,
                           stream=None, check=True) -> int:
    """Block-sparse forward; block_mask is a device uint8 [mask_heads, nt, nt]
    buffer (nt = ceil(N / 128)), mask_heads 1 or H."""
    st = _lib.fa_forward_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                     float(scale), int(bool(causal)), _ptr(block_mask),
                                     int(mask_heads), _stream(stream))
    return _check(st, "fa_forward_blocksparse", check)


def fa_backward_blocksparse(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal,
                            block_mask, mask_heads, workspace, workspace_bytes, stream=None,
                            check=True) -> int:
    st = _lib.fa_backward_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                      _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                      int(bool(causal)), _ptr(block_mask), int(mask_heads),
                                      _ptr(workspace), int(workspace_bytes), _stream(stream))
    return _check(st, "fa_backward_blocksparse", check)


def fa_forward_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, num_splits, workspace,
                       workspace_bytes, stream=None, check=True) -> int:
    st = _lib.fa_forward_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                                 float(scale), int(bool(causal)), int(num_splits),
                                 _ptr(workspace), int(workspace_bytes), _stream(stream))
    return _check(st, "fa_forward_splitkv", check)


def fa_splitkv_default_splits(B, H, Nq, Nk) -> int:
    return int(_lib.fa_splitkv_default_splits(B, H, Nq, Nk))


def fa_splitkv_workspace_size(B, H, Nq, Nk, d, num_splits) -> int:
    return int(_lib.fa_splitkv_workspace_size(B, H, Nq, Nk, d, num_splits))


def fa_forward_fp8(q8, k8, v8, q_descale, k_descale, v_descale, o, lse, B, H, N, d, scale,
                   causal, stream=None, check=True) -> int:
    """FP8 forward: q8, k8, v8 are E4M3 codes (uint8 or float8_e4m3fn device
    tensors), the descales device fp32 scalars or None (= 1)."""
    st = _lib.fa_forward_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_descale), _ptr(k_descale),
                             _ptr(v_descale), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                             int(bool(causal)), _stream(stream))
    return _check(st, "fa_forward_fp8", check)


def fa_quantize_fp8(x, dtype, n, codes, descale, stream=None, check=True) -> int:
    """Per-tensor E4M3 quantisation of n elements of x (FA_BF16 or FA_FP32)
    into codes (n bytes) and descale (one device fp32)."""
    st = _lib.fa_quantize_fp8(_ptr(x), int(dtype), int(n), _ptr(codes), _ptr(descale),
                              _stream(stream))
    return _check(st, "fa_quantize_fp8", check)
