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


def _block_mask(block_mask: torch.Tensor, H: int, N: int, device) -> Tuple[torch.Tensor, int]:
    """Validate a block mask: bool/uint8 [nt, nt] or [Hm, nt, nt] (Hm = 1 or
    H), nt = ceil(N / 128); returns a contiguous uint8 device copy and Hm."""
    nt = (N + 127) // 128
    m = block_mask if block_mask.dim() == 3 else block_mask.unsqueeze(0)
    if m.dim() != 3 or tuple(m.shape[1:]) != (nt, nt) or m.shape[0] not in (1, H):
        raise ValueError(f"block_mask must be [nt, nt] or [1 or H, nt, nt] with nt = {nt}")
    m = m.to(device=device, dtype=torch.uint8).contiguous()
    return m, int(m.shape[0])


def attention_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      scale: Optional[float] = None, causal: bool = False,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      block_mask: Optional[torch.Tensor] = None
                      ) -> Tuple[torch.Tensor, torch.Tensor]:
    """O and LSE.  With ``block_mask`` (bf16 only): block-sparse attention over
    128 x 128 tiles, see ``fa_forward_blocksparse``."""
    _check_inputs(q, k, v)
    B, H, N, d = _dims(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    if block_mask is not None:
        m, mh = _block_mask(block_mask, H, N, q.device)
        nat.fa_forward_blocksparse(q, k, v, out, lse, B, H, N, d, scale, causal, m, mh)
    else:
        nat.fa_forward_ex(q, k, v, out, lse, B, H, N, d, scale, causal, _dtype_code(q))
    return out, lse


def attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                       do: torch.Tensor, lse: torch.Tensor, scale: Optional[float] = None,
                       causal: bool = False, workspace: Optional[torch.Tensor] = None,
                       block_mask: Optional[torch.Tensor] = None
                       ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """dQ, dK, dV; ``block_mask`` as in ``attention_forward`` (same mask as the
    forward)."""
    _check_inputs(q, k, v, o, do)
    B, H, N, d = _dims(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    wbytes = nat.fa_backward_workspace_size(B, H, N, d)
    if workspace is None or workspace.numel() * workspace.element_size() < wbytes:
        workspace = torch.empty(wbytes, device=q.device, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if block_mask is not None:
        m, mh = _block_mask(block_mask, H, N, q.device)
        nat.fa_backward_blocksparse(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, scale, causal,
                                    m, mh, workspace, wbytes)
    else:
        nat.fa_backward_ex(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, scale, causal,
                           workspace, wbytes, _dtype_code(q))
    return dq, dk, dv


def attention_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                     scale: Optional[float] = None, causal: bool = False,
                     num_splits: Optional[int] = None
                     ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV forward (bf16): q [B, H, N_q, d] against k, v [B, H, N_k, d];
    see ``fa_forward_splitkv``.  Returns O [B, H, N_q, d] and LSE [B, H, N_q]."""
    _check_inputs(k, v)
    if not q.is_cuda or not q.is_contiguous() or q.dtype != k.dtype or q.dim() != 4 \
            or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise ValueError("q must be a contiguous CUDA [B, H, N_q, d] tensor matching k and v")
    B, H, Nq, d = _dims(q)
    Nk = int(k.shape[2])
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    s = nat.fa_splitkv_default_splits(B, H, Nq, Nk) if num_splits is None else int(num_splits)
    wbytes = nat.fa_splitkv_workspace_size(B, H, Nq, Nk, d, s)
    ws = torch.empty(wbytes, device=q.device, dtype=torch.uint8)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32)
    nat.fa_forward_splitkv(q, k, v, out, lse, B, H, Nq, Nk, d, scale, causal, s, ws, wbytes)
    return out, lse


def _codes(t: torch.Tensor) -> torch.Tensor:
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise ValueError("E4M3 inputs must be uint8 codes or float8_e4m3fn tensors")
    return t


def _descale(x, device) -> Optional[torch.Tensor]:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        if not x.is_cuda or x.dtype != torch.float32 or x.numel() != 1:
            raise ValueError("a descale tensor must be one fp32 element on the GPU")
        return x
    return torch.tensor([float(x)], device=device, dtype=torch.float32)


def quantize_fp8(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-tensor E4M3 quantisation of a contiguous bf16 or fp32 CUDA tensor
    (see ``fa_quantize_fp8``): returns the codes (uint8, x's shape) and the
    descale factor (a one-element fp32 CUDA tensor, amax / 448)."""
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    codes = torch.empty(x.shape, device=x.device, dtype=torch.uint8)
    descale = torch.empty(1, device=x.device, dtype=torch.float32)
    nat.fa_quantize_fp8(x, _dtype_code(x), x.numel(), codes, descale)
    return codes, descale


def attention_forward_fp8(q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor,
                          q_descale=None, k_descale=None, v_descale=None,
                          scale: Optional[float] = None, causal: bool = False,
                          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """FP8 forward (see ``fa_forward_fp8``): E4M3 q8, k8, v8 [B, H, N, d]
    (uint8 codes or float8_e4m3fn), per-tensor descale factors (one-element
    fp32 CUDA tensors, python floats, or None for 1).  Returns O (bf16) and
    LSE (fp32)."""
    for t in (q8, k8, v8):
        _codes(t)
        if not t.is_cuda or not t.is_contiguous() or t.shape != q8.shape:
            raise ValueError("inputs must be contiguous CUDA tensors of one shape")
    B, H, N, d = _dims(q8)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = (_descale(x, q8.device) for x in (q_descale, k_descale, v_descale))
    if out is None:
        out = torch.empty((B, H, N, d), device=q8.device, dtype=torch.bfloat16)
    if lse is None:
        lse = torch.empty((B, H, N), device=q8.device, dtype=torch.float32)
    nat.fa_forward_fp8(q8, k8, v8, dq, dk, dv, out, lse, B, H, N, d, scale, causal)
    return out, lse
