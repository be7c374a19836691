"""Host-side checks that need no GPU: the C-ABI library loads and exports
every entry point the header declares, argument errors are reported before
anything touches a device, the workspace formula is linear in N, and the
benchmark's FLOP counter reproduces the page's worked numbers."""
import ctypes
import os
import re

import pytest

import workloads
from exact_io_aware_99_b200 import perf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def _lib():
    import exact_io_aware_99_b200 as fa
    return fa


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("fa_forward", "fa_backward", "fa_backward_workspace_size", "fa_status_string"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    fa = _lib()
    lib = ctypes.CDLL(fa.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(fa.EXPORTS)


def test_status_strings():
    fa = _lib()
    assert fa.fa_status_string(0) == "ok"
    for code in (-1, -2, -3, -4, -5, -6):
        s = fa.fa_status_string(code)
        assert s and s != "unknown status"
    assert fa.fa_status_string(12345) == "unknown status"


# Each of these must be rejected before any CUDA call (so they pass on a
# machine without a GPU).  Pointers are fake but 256-byte aligned.
A = 1 << 20


@pytest.mark.parametrize("args,code", [
    (dict(q=0), -1),                     # null pointer
    (dict(B=0), -1), (dict(H=0), -1), (dict(N=0), -1),   # empty problem
    (dict(scale=0.0), -1), (dict(scale=float("nan")), -1), (dict(scale=-1.0), -1),
    (dict(d=96), -2), (dict(d=32), -2), (dict(d=256), -2),
    (dict(q=A + 8), -3), (dict(o=A + 4), -3), (dict(lse=A + 2), -3),
])
def test_forward_argument_errors(args, code):
    fa = _lib()
    kw = dict(q=A, k=2 * A, v=3 * A, o=4 * A, lse=5 * A, B=1, H=2, N=256, d=64, scale=0.125)
    kw.update(args)
    st = fa.fa_forward(kw["q"], kw["k"], kw["v"], kw["o"], kw["lse"], kw["B"], kw["H"],
                       kw["N"], kw["d"], kw["scale"], 0, stream=0, check=False)
    assert st == code


def test_fp32_path_accepts_any_small_head_dim_but_not_above_128():
    fa = _lib()
    st = fa.fa_forward_ex(A, 2 * A, 3 * A, 4 * A, 5 * A, 1, 1, 16, 129, 0.1, 0, fa.FA_FP32,
                          stream=0, check=False)
    assert st == fa.FA_ERR_UNSUPPORTED
    st = fa.fa_forward_ex(A, 2 * A, 3 * A, 4 * A, 5 * A, 1, 1, 16, 7, 0.1, 0, 7,
                          stream=0, check=False)
    assert st == fa.FA_ERR_UNSUPPORTED


@pytest.mark.parametrize("ws_ptr,ws_bytes,code", [
    (0, 1 << 30, -4),            # null workspace
    (A, 16, -4),                 # too small
    (A + 16, 1 << 30, -4),       # not 256-byte aligned
])
def test_backward_workspace_errors(ws_ptr, ws_bytes, code):
    fa = _lib()
    st = fa.fa_backward(A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 7 * A, 8 * A, 9 * A, 1, 2, 256, 64,
                        0.125, 1, ws_ptr, ws_bytes, stream=0, check=False)
    assert st == code


def test_workspace_size_is_linear_in_n():
    fa = _lib()
    sizes = [fa.fa_backward_workspace_size(2, 4, n, 128) for n in (1024, 2048, 4096, 8192)]
    diffs = [b - a for a, b in zip(sizes, sizes[1:])]
    # doubling N doubles the increment: linear, not quadratic
    assert diffs[1] == 2 * diffs[0] and diffs[2] == 2 * diffs[1]
    # two fp32 row vectors (D and the base-2 LSE) padded to 128-row tiles,
    # each rounded to 256 bytes
    B, H, N, d = 2, 4, 1000, 80
    np_ = 1024
    up = lambda x: (x + 255) // 256 * 256
    assert fa.fa_backward_workspace_size(B, H, N, d) == 2 * up(4 * B * H * np_)
    assert fa.fa_backward_workspace_size(0, 1, 1, 64) == 0


def test_flop_counter_matches_the_pages_worked_numbers():
    # "FlashAttention-2" review, implementation-cost answer, (1) FLOPs:
    # N = 1024, d = 64 -> forward 268,435,456, backward 671,088,640, total ~939e6.
    assert perf.fwd_flops(1, 1, 1024, 64, False) == 268_435_456
    assert perf.bwd_flops(1, 1, 1024, 64, False) == 671_088_640
    total = perf.fwd_flops(1, 1, 1024, 64, False) + perf.bwd_flops(1, 1, 1024, 64, False)
    assert int(total // 1e6) == 939  # 939.5e6, printed as "about 939 x 10^6"
    assert perf.fwd_flops(1, 1, 1024, 64, True) == 268_435_456 / 2


def test_workload_table():
    w = workloads.WORKLOADS["causal_d128"]
    assert (w.B, w.H, w.N, w.d, w.causal, w.backward) == (4, 16, 4096, 128, True, True)
    assert abs(perf.fwd_flops(w.B, w.H, w.N, w.d, True) - 274.9e9) < 0.1e9
    assert abs(perf.bwd_flops(w.B, w.H, w.N, w.d, True) - 687.2e9) < 0.1e9
    w5 = workloads.WORKLOADS["gpt3_d80"]
    assert w5.H * w5.d == w5.hidden == 2560


def test_inputs_are_seeded_and_rounded():
    w = workloads.WORKLOADS["fwd_d64"]
    a = workloads.make_inputs(w, B=1, H=1, N=64)
    b = workloads.make_inputs(w, B=1, H=1, N=64)
    import torch
    assert a["q"].dtype == torch.bfloat16
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["v"], b["v"])
    p = workloads.make_inputs(workloads.WORKLOADS["gpt3_d80"], B=1, H=2, N=16)
    assert p["q"].shape == (1, 2, 16, 80)
    # projections of unit normals through N(0, 0.02^2) 2560-wide weights:
    # entries have variance about 2560 * 0.02^2 = 1.02
    big = workloads.make_inputs(workloads.WORKLOADS["gpt3_d80"], B=1, H=32, N=64)
    var = big["k"].float().var().item()
    assert 0.85 < var < 1.2


def test_masked_flop_counts_reduce_to_the_dense_ones():
    import numpy as np
    from exact_io_aware_99_b200 import perf
    for N in (1, 127, 128, 300, 1000):
        nt = (N + 127) // 128
        ones = np.ones((nt, nt), bool)
        for causal in (False, True):
            dense = N * (N + 1) / 2 if causal else float(N * N)
            assert perf.visible_pairs(ones, N, causal) == dense
        # masked flops of an all-ones mask = the dense count (H heads shared)
        assert perf.fwd_flops_masked(2, 3, N, 64, False, ones) == perf.fwd_flops(2, 3, N, 64, False)
    # one visible interior block of a 3 x 3 mask: 128 x 128 pairs
    m = np.zeros((3, 3), bool)
    m[1, 0] = True
    assert perf.visible_pairs(m, 300, False) == 128 * 128
    # per-head masks are counted per head
    mh = np.zeros((2, 3, 3), bool)
    mh[0, 1, 0] = mh[1, 2, 2] = True           # tile 2 is 44 rows: 44 x 44
    assert perf.fwd_flops_masked(1, 2, 300, 8, False, mh) == 4 * 8 * (128 * 128 + 44 * 44)


def test_splitkv_workspace_formula_and_split_clamping():
    fa = _lib()
    up = lambda x: (x + 255) // 256 * 256
    # 3 splits of a 1000-key cache (8 key tiles -> ranges of 3, 3, 2 tiles)
    B, H, Nq, Nk, d = 2, 3, 5, 1000, 80
    rows = 3 * B * H * Nq
    assert fa.fa_splitkv_workspace_size(B, H, Nq, Nk, d, 3) == up(rows * d * 4) + up(rows * 4)
    # more splits than key tiles clamp to one tile per split; 5 requested
    # splits of 8 tiles become ranges of 2 tiles, i.e. 4 splits
    assert fa.fa_splitkv_workspace_size(1, 1, 16, 256, 128, 10) == \
        fa.fa_splitkv_workspace_size(1, 1, 16, 256, 128, 2)
    assert fa.fa_splitkv_workspace_size(1, 1, 16, 1024, 128, 5) == \
        fa.fa_splitkv_workspace_size(1, 1, 16, 1024, 128, 4)
    for bad in ((0, 1, 1, 1, 64, 1), (1, 1, 0, 1, 64, 1), (1, 1, 1, 0, 64, 1),
                (1, 1, 1, 1, 64, 0), (1, 1, 1, 1, 200, 1)):
        assert fa.fa_splitkv_workspace_size(*bad) == 0
    assert 1 <= fa.fa_splitkv_default_splits(1, 1, 1, 16384) <= 128
    assert fa.fa_splitkv_default_splits(1, 1, 1, 100) == 1


def test_new_entry_points_reject_bad_arguments_before_any_device_call():
    fa = _lib()
    # split-KV: null pointer, zero splits, bad head dim
    st = fa.fa_forward_splitkv(0, A, A, A, A, 1, 1, 4, 256, 64, 0.1, 0, 1, A, 1 << 20,
                               stream=0, check=False)
    assert st == -1
    st = fa.fa_forward_splitkv(A, A, A, A, A, 1, 1, 4, 256, 64, 0.1, 0, 0, A, 1 << 20,
                               stream=0, check=False)
    assert st == -1
    st = fa.fa_forward_splitkv(A, A, A, A, A, 1, 1, 4, 256, 96, 0.1, 0, 1, A, 1 << 20,
                               stream=0, check=False)
    assert st == -2
    # block-sparse: null mask, mask_heads neither 1 nor H
    st = fa.fa_forward_blocksparse(A, A, A, A, A, 1, 2, 256, 64, 0.1, 0, None, 1, stream=0, check=False)
    assert st == -1
    st = fa.fa_forward_blocksparse(A, A, A, A, A, 1, 2, 256, 64, 0.1, 0, A, 3, stream=0, check=False)
    assert st == -1
    st = fa.fa_backward_blocksparse(A, A, A, A, A, A, A, A, A, 1, 2, 256, 64, 0.1, 0, A, 5,
                                    A, 1 << 20, stream=0, check=False)
    assert st == -1


def test_decode_flop_and_byte_counts():
    assert perf.decode_pairs(3, 7, True) == 5 + 6 + 7
    assert perf.decode_pairs(5, 3, True) == 0 + 0 + 1 + 2 + 3
    assert perf.decode_pairs(4, 9, False) == 36
    # square causal decode = the dense causal pair count N (N + 1) / 2
    assert perf.decode_pairs(300, 300, True) == 300 * 301 / 2
    assert perf.decode_flops(2, 3, 4, 9, 16, False) == 4 * 16 * 2 * 3 * 36
    assert perf.decode_bytes(1, 1, 2, 10, 8) == 2 * 2 * 8 * 2 + 2 * 10 * 8 * 2 + 4 * 2


def test_fp8_entry_points_reject_bad_arguments_before_any_device_call():
    fa = _lib()
    # null input, unsupported head dim, misaligned code or descale pointers
    st = fa.fa_forward_fp8(0, A, A, None, None, None, A, A, 1, 1, 128, 64, 0.1, 0,
                           stream=0, check=False)
    assert st == -1
    st = fa.fa_forward_fp8(A, A, A, None, None, None, A, A, 1, 1, 128, 96, 0.1, 0,
                           stream=0, check=False)
    assert st == -2
    st = fa.fa_forward_fp8(A + 8, A, A, None, None, None, A, A, 1, 1, 128, 64, 0.1, 0,
                           stream=0, check=False)
    assert st == -3
    st = fa.fa_forward_fp8(A, A, A, A + 2, None, None, A, A, 1, 1, 128, 64, 0.1, 0,
                           stream=0, check=False)
    assert st == -3
    st = fa.fa_forward_fp8(A, A, A, None, None, None, A, A, 1, 1, 0, 64, 0.1, 0,
                           stream=0, check=False)
    assert st == -1
    # quantiser: empty input, unknown dtype, misaligned codes
    assert fa.fa_quantize_fp8(A, fa.FA_BF16, 0, A, A, stream=0, check=False) == -1
    assert fa.fa_quantize_fp8(A, 9, 16, A, A, stream=0, check=False) == -2
    assert fa.fa_quantize_fp8(A, fa.FA_FP32, 16, A + 4, A, stream=0, check=False) == -3


def test_fp8_workload_and_generators():
    import torch
    w = workloads.WORKLOADS["fp8_causal_d128"]
    assert (w.B, w.H, w.N, w.d, w.dtype, w.causal, w.backward) == \
        (4, 16, 4096, 128, "e4m3", True, False)
    a = workloads.make_fp8_inputs(w, B=1, H=1, N=64)
    b = workloads.make_fp8_inputs(w, B=1, H=1, N=64)
    assert a["q8"].dtype == torch.uint8 and a["q8"].shape == (1, 1, 64, 128)
    assert torch.equal(a["k8"], b["k8"]) and a["v_descale"] == b["v_descale"]
    # the largest magnitude of each tensor maps onto 448 (code 0x7E / 0xFE)
    for n in ("q8", "k8", "v8"):
        assert int((a[n] & 0x7F).max()) == 0x7E


def test_fp8_step_counts_only_the_forward():
    import bench
    w = workloads.WORKLOADS["fp8_causal_d128"]
    f, b = bench.step_flop_counts(w)
    assert b == 0.0
    assert f == perf.fwd_flops(4, 16, 4096, 128, True)
    assert abs(f - 274.9e9) < 0.1e9


def test_forward_key_tile_table_and_override():
    # host-side logic only: the table picks the 64-key kernel for short causal
    # problems, the override forces either kernel, bad sizes are rejected
    m = _lib()
    assert m.fa_forward_key_tile(128, 256, True) == 64
    assert m.fa_forward_key_tile(128, 257, True) == 128
    assert m.fa_forward_key_tile(80, 200, True) == 64
    assert m.fa_forward_key_tile(80, 512, True) == 64
    assert m.fa_forward_key_tile(80, 513, True) == 128
    assert m.fa_forward_key_tile(64, 512, True) == 64
    assert m.fa_forward_key_tile(64, 513, True) == 128
    assert m.fa_forward_key_tile(128, 128, False) == 128
    assert m.fa_forward_key_tile(96, 128, True) == 0
    assert m.fa_forward_key_tile(128, 0, True) == 0
    assert m.fa_set_forward_key_tile(7, check=False) == m.FA_ERR_INVALID_ARG
    try:
        m.fa_set_forward_key_tile(128)
        assert m.fa_forward_key_tile(128, 256, True) == 128
        m.fa_set_forward_key_tile(64)
        assert m.fa_forward_key_tile(128, 16384, False) == 64
    finally:
        m.fa_set_forward_key_tile(0)
    assert m.fa_forward_key_tile(128, 16384, False) == 128


def test_profile_source_hash_ignores_comments_only():
    # a profile's recorded traffic stays valid across comment edits of the
    # kernel sources, and not across code edits
    import bench
    code = "int a = 1; // one\n/* block\n comment */\nint b = a + 2;\n"
    assert bench._code_only(code) == bench._code_only("int a = 1;\n\nint b = a + 2; // two\n")
    assert bench._code_only(code) != bench._code_only("int a = 1;\nint b = a + 3;\n")
