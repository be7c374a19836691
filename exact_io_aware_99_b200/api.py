"""Tensor-level wrappers over the C ABI: allocate outputs with torch and call
the library on the current stream.  Inputs must be contiguous [B, H, N, d]
CUDA tensors of one dtype (bf16, or fp32 for the fp32 path)."""
from __future__ import annotations

import math
from typing import Optional, Tuple

import torch

from . import _native as nat


def _dims(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return nat.FA_BF16
    if t.dtype == torch.float32:
        return nat.FA_FP32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _check_inputs(*ts: torch.Tensor):
    ref = ts[0]
    for t in ts:
        if not t.is_cuda or not t.is_contiguous() or t.dtype != ref.dtype or t.shape != ref.shape:
            raise ValueError("inputs must be contiguous CUDA tensors of one shape and dtype")


def attention_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      scale: Optional[float] = None, causal: bool = False,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None
                      ) -> Tuple[torch.Tensor, torch.Tensor]:
    _check_inputs(q, k, v)
    B, H, N, d = _dims(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    nat.fa_forward_ex(q, k, v, out, lse, B, H, N, d, scale, causal, _dtype_code(q))
    return out, lse


def attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                       do: torch.Tensor, lse: torch.Tensor, scale: Optional[float] = None,
                       causal: bool = False, workspace: Optional[torch.Tensor] = None
                       ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    _check_inputs(q, k, v, o, do)
    B, H, N, d = _dims(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    wbytes = nat.fa_backward_workspace_size(B, H, N, d)
    if workspace is None or workspace.numel() * workspace.element_size() < wbytes:
        workspace = torch.empty(wbytes, device=q.device, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nat.fa_backward_ex(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace,
                       wbytes, _dtype_code(q))
    return dq, dk, dv
