"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the attention arithmetic, so both the fp64 CPU oracle and
the CUDA path can take their inputs from here without sharing any of the
method's code.

Workloads (shapes are [B, H, N, d], d fastest):

* ``fp32_small``  B1 H2 N256 d64, fp32, forward only, non-causal.
* ``fwd_d64``     B8 H16 N1024 d64, bf16, forward only, non-causal.
* ``causal_d128`` B4 H16 N4096 d128, bf16, causal, forward+backward.
* ``long_d128``   B1 H16 N16384 d128, bf16, causal, forward+backward.
* ``bsparse_d128`` B1 H16 N16384 d128, bf16, non-causal, forward+backward,
  block-sparse: every query tile sees the key tiles within 4 tiles of its
  own plus key tiles 0 and 1 (a local window with global tokens, the hybrid
  local + global pattern the FlashAttention-2 review names for sparse
  attention); 128 x 128 tiles, one mask for all heads, ~8.6 % of the pairs.
* ``decode_d128`` B8 H16, 128 new queries against a 16384-entry key/value
  cache, d128, bf16, causal (the queries are the last 128 positions),
  forward only, split-KV.
* ``gpt3_d80``    B8 H32 N2048 d80, bf16, causal, forward+backward; Q, K, V
  are projections X.W of a unit-normal activation X [B, N, 2560] through
  three independent N(0, 0.02^2) [2560, 2560] weights, then split into
  32 heads of 80 (the GPT-3 2.7B layer shape named on the FlashAttention-2
  review page, section on results, GPT-3 2.7B end-to-end training).
* ``fp8_causal_d128`` B4 H16 N4096 d128, E4M3 Q/K/V with one fp32
  dequantisation factor per tensor, causal, forward only (the FP8 forward the
  FlashAttention-2 review lists under future work, item (5)); the same shape
  as ``causal_d128``.

Every tensor is generated in fp32 on the CPU from ``torch.Generator`` seeded
with ``1000 + index`` and then rounded (round-to-nearest-even) to the storage
dtype, so the GPU and the oracle see the same bits.  E4M3 tensors are drawn
the same way in fp32 and then quantised per tensor by ``quantize_e4m3``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    N: int
    d: int
    dtype: str          # "fp32", "bf16" or "e4m3"
    causal: bool
    backward: bool
    projected: bool = False   # Q/K/V = X.W (GPT-3 shaped layer)
    hidden: int = 0
    mask: str = ""            # block-sparse pattern name ("" = dense)
    nk: int = 0               # keys when they differ from the N queries (decode)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"fp32": torch.float32, "bf16": torch.bfloat16,
                "e4m3": torch.float8_e4m3fn}[self.dtype]

    def describe(self) -> str:
        pas = "fwd+bwd" if self.backward else "fwd"
        cz = "causal" if self.causal else "non-causal"
        bs = f" block-sparse {self.mask}" if self.mask else ""
        n = f"N_q{self.N} N_k{self.nk}" if self.nk else f"N{self.N}"
        return (f"{self.name}: B{self.B} H{self.H} {n} d{self.d} "
                f"{self.dtype} {cz}{bs} {pas}")


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("fp32_small", 0, 1, 2, 256, 64, "fp32", False, False),
        Workload("fwd_d64", 1, 8, 16, 1024, 64, "bf16", False, False),
        Workload("causal_d128", 2, 4, 16, 4096, 128, "bf16", True, True),
        Workload("long_d128", 3, 1, 16, 16384, 128, "bf16", True, True),
        Workload("gpt3_d80", 4, 8, 32, 2048, 80, "bf16", True, True,
                 projected=True, hidden=2560),
        Workload("bsparse_d128", 5, 1, 16, 16384, 128, "bf16", False, True,
                 mask="local4_global2"),
        Workload("decode_d128", 6, 8, 16, 128, 128, "bf16", True, False, nk=16384),
        Workload("fp8_causal_d128", 7, 4, 16, 4096, 128, "e4m3", True, False),
    ]
}


def block_mask(w: Workload, N: Optional[int] = None):
    """The workload's block mask as numpy bool [1, nt, nt] (128-row tiles),
    or None for a dense workload.  ``local4_global2``: query tile I sees key
    tiles J with |I - J| <= 4, and key tiles 0 and 1."""
    import numpy as np
    if not w.mask:
        return None
    N = w.N if N is None else N
    nt = (N + 127) // 128
    if w.mask == "local4_global2":
        i = np.arange(nt)
        m = np.abs(i[:, None] - i[None, :]) <= 4
        m[:, :2] = True
        return m[None]
    raise ValueError(f"unknown mask pattern {w.mask}")


def round_to(x: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    """Round an fp32 tensor to ``dtype`` (RNE) and keep it in that dtype."""
    return x.to(dtype).contiguous()


def randn(shape, seed: int, dtype: torch.dtype = torch.bfloat16,
          std: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return round_to(x, dtype)


def make_inputs(w: Workload, with_grad_out: Optional[bool] = None,
                B: Optional[int] = None, H: Optional[int] = None,
                N: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Seeded CPU inputs for workload ``w``.

    B/H/N may be overridden to draw a smaller instance with the same
    distribution (used by sampled and reduced-size checks).  Returns q, k,
    v (and do when a backward is requested), contiguous [B, H, N, d].
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    want_do = w.backward if with_grad_out is None else with_grad_out
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    dt = w.torch_dtype
    out: Dict[str, torch.Tensor] = {}
    if w.projected:
        hid = w.hidden
        hid_eff = H * w.d
        x = torch.randn(B, N, hid, generator=g, dtype=torch.float32)
        for name in ("q", "k", "v"):
            wmat = torch.randn(hid, hid_eff, generator=g, dtype=torch.float32) * 0.02
            proj = torch.matmul(x, wmat)                      # [B, N, H*d] fp32
            proj = proj.view(B, N, H, w.d).permute(0, 2, 1, 3).contiguous()
            out[name] = round_to(proj, dt)
    else:
        for name in ("q", "k", "v"):
            out[name] = round_to(
                torch.randn(B, H, N, w.d, generator=g, dtype=torch.float32), dt)
    if want_do:
        out["do"] = round_to(
            torch.randn(B, H, N, w.d, generator=g, dtype=torch.float32), dt)
    return out


def random_case(B: int, H: int, N: int, d: int, seed: int,
                dtype: torch.dtype = torch.bfloat16, grad: bool = True,
                std: float = 1.0) -> Dict[str, torch.Tensor]:
    """Small seeded iid-normal case (parity tests at odd sizes)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    out = {}
    names = ("q", "k", "v", "do") if grad else ("q", "k", "v")
    for name in names:
        x = torch.randn(B, H, N, d, generator=g, dtype=torch.float32) * std
        out[name] = round_to(x, dtype)
    return out


def make_decode_inputs(w: Workload, B: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Seeded CPU inputs of a decode workload: q [B, H, N, d] and k, v
    [B, H, nk, d], iid N(0, 1) rounded to the storage dtype."""
    B = w.B if B is None else B
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    dt = w.torch_dtype
    out = {"q": round_to(torch.randn(B, w.H, w.N, w.d, generator=g), dt)}
    for name in ("k", "v"):
        out[name] = round_to(torch.randn(B, w.H, w.nk, w.d, generator=g), dt)
    return out


# Largest finite E4M3 value (1.75 * 2^8); the per-tensor quantisation maps
# the tensor's largest magnitude onto it.
E4M3_MAX = 448.0


def quantize_e4m3(x: torch.Tensor) -> Tuple[torch.Tensor, float]:
    """Per-tensor E4M3 quantisation of a float tensor (computed in fp32):
    amax = max |x|, descale = amax / 448 and codes = RN(x * (448 / amax)),
    each step one fp32 operation, the last through torch's float8_e4m3fn
    conversion (round to nearest even).  When 448 / amax has no finite fp32
    value (amax = 0, or amax below about 1.3e-36) the tensor is taken as it
    is: factor 1, descale 1.  Returns the codes as a contiguous uint8 tensor
    and the fp32 descale factor."""
    xf = x.float()
    amax = xf.abs().max() if xf.numel() else torch.tensor(0.0)
    lim = torch.tensor(E4M3_MAX, dtype=torch.float32)
    inv = lim / amax if float(amax) > 0.0 else torch.tensor(float("inf"))
    if bool(torch.isfinite(inv)):
        descale = float(amax / lim)
    else:
        inv = torch.tensor(1.0, dtype=torch.float32)
        descale = 1.0
    codes = (xf * inv).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    return codes, descale


def make_fp8_inputs(w: Workload, B: Optional[int] = None, H: Optional[int] = None,
                    N: Optional[int] = None, seed: Optional[int] = None) -> Dict[str, object]:
    """Seeded inputs of an E4M3 workload: q, k, v drawn iid N(0, 1) in fp32
    [B, H, N, d] and quantised per tensor.  Returns {"q8", "k8", "v8"} (uint8
    codes) and {"q_descale", "k_descale", "v_descale"} (floats)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    g = torch.Generator(device="cpu").manual_seed(w.seed if seed is None else seed)
    out: Dict[str, object] = {}
    for name in ("q", "k", "v"):
        codes, ds = quantize_e4m3(torch.randn(B, H, N, w.d, generator=g, dtype=torch.float32))
        out[name + "8"] = codes
        out[name + "_descale"] = ds
    return out


def fp8_random_case(B: int, H: int, N: int, d: int, seed: int,
                    std: float = 1.0) -> Dict[str, object]:
    """Small seeded E4M3 case (iid N(0, std^2), quantised per tensor)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    out: Dict[str, object] = {}
    for name in ("q", "k", "v"):
        codes, ds = quantize_e4m3(torch.randn(B, H, N, d, generator=g) * std)
        out[name + "8"] = codes
        out[name + "_descale"] = ds
    return out


def fp8_exact_case(B: int, H: int, N: int, d: int, seed: int) -> Dict[str, object]:
    """E4M3 case whose probabilities are exact E4M3 values.

    Every query row holds one or two entries of +-1 (code value; descale
    1/2), every key entry is an integer in [-2, 2] (descale 2), so with the
    attention scale ln 2 each score, in base-2 units, is an integer in
    [-4, 4]: any probability taken against a reference maximum inside the
    row's range is a power of two between 2^-8 and 2^8, which E4M3 holds
    exactly.  V is iid N(0, 1) quantised per tensor.  Use scale = ln 2."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.zeros(B, H, N, d)
    nnz = torch.randint(1, 3, (B, H, N), generator=g)
    pos = torch.randint(0, d, (B, H, N, 2), generator=g)
    sgn = torch.randint(0, 2, (B, H, N, 2), generator=g).float() * 2 - 1
    for t in range(2):
        keep = (nnz > t).float()
        q.scatter_add_(3, pos[..., t:t + 1], (sgn[..., t] * keep).unsqueeze(-1))
    q = q.clamp(-1.0, 1.0)   # two hits on one position stay within +-1
    k = torch.randint(-2, 3, (B, H, N, d), generator=g).float()
    v8, v_ds = quantize_e4m3(torch.randn(B, H, N, d, generator=g))
    return {
        "q8": q.to(torch.float8_e4m3fn).view(torch.uint8).contiguous(),
        "k8": k.to(torch.float8_e4m3fn).view(torch.uint8).contiguous(),
        "v8": v8,
        "q_descale": 0.5, "k_descale": 2.0, "v_descale": v_ds,
    }
