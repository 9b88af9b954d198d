"""The C-ABI library without a GPU: it loads, exports every declared entry
point, and rejects invalid arguments synchronously (nothing is launched on
these paths, so no device is needed)."""
import ctypes
import os
import re

import pytest

import attention_gqa_decode_b200 as gqa
from attention_gqa_decode_b200 import _lib
from attention_gqa_decode_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return gqa.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gqa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(gqa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted(_lib.SIGNATURES)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert isinstance(getattr(L, name), ctypes._CFuncPtr), name


def test_status_strings(L):
    for code in range(5):
        assert gqa.gqa_status_string(code).startswith("GQA_")
    assert "unknown" in gqa.gqa_status_string(99)


A = 1 << 20        # a 16-byte-aligned fake address; never dereferenced on these paths
BAD = A + 2        # misaligned


@pytest.mark.parametrize("args,expect", [
    # q, k, v, out, B, S_q, S_kv, h, n_kv, d, causal, scale
    ((0, A, A, A, 1, 8, 8, 4, 1, 64, 1, 0.125), _lib.GQA_ERR_INVALID_ARG),     # null pointer
    ((A, BAD, A, A, 1, 8, 8, 4, 1, 64, 1, 0.125), _lib.GQA_ERR_INVALID_ARG),   # misaligned
    ((A, A, A, A, 0, 8, 8, 4, 1, 64, 1, 0.125), _lib.GQA_ERR_INVALID_ARG),     # B = 0
    ((A, A, A, A, 1, 0, 8, 4, 1, 64, 1, 0.125), _lib.GQA_ERR_INVALID_ARG),     # S_q = 0
    ((A, A, A, A, 1, 8, -1, 4, 1, 64, 1, 0.125), _lib.GQA_ERR_INVALID_ARG),    # S_kv < 0
    ((A, A, A, A, 1, 8, 8, 6, 4, 64, 1, 0.125), _lib.GQA_ERR_INVALID_ARG),     # h % n_kv != 0
    ((A, A, A, A, 1, 9, 8, 4, 1, 64, 1, 0.125), _lib.GQA_ERR_INVALID_ARG),     # causal, S_q > S_kv
    ((A, A, A, A, 1, 8, 8, 4, 1, 64, 1, float("nan")), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, 1, 8, 8, 4, 1, 64, 1, float("inf")), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, 1, 8, 8, 4, 1, 64, 1, -0.5), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, 1, 8, 8, 4, 1, 96, 1, 0.125), _lib.GQA_ERR_UNSUPPORTED),     # d_h = 96
    ((A, A, A, A, 1, 8, 8, 4, 1, 256, 0, 0.125), _lib.GQA_ERR_UNSUPPORTED),
])
def test_prefill_rejects(L, args, expect):
    assert gqa.gqa_prefill(*args, None) == expect


@pytest.mark.parametrize("args,expect", [
    # q, k, v, seqlens, out, B, h, n_kv, d, scale
    ((A, A, A, 0, A, 2, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),       # null seqlens
    ((A, A, A, A + 1, A, 2, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),   # misaligned seqlens
    ((A, A, BAD, A, A, 2, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, 0, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, 65536, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),   # B above the grid limit
    ((A, A, A, A, A, 2, 4, 3, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, 2, 0, 1, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, 2, 4, 2, 128, float("nan")), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, 2, 4, 2, 32, 0.1), _lib.GQA_ERR_UNSUPPORTED),
])
def test_decode_rejects(L, args, expect):
    assert gqa.gqa_decode(*args, None) == expect


def test_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gqa.prefill(q, q[:, :, :1].contiguous(), q[:, :, :1].contiguous())
    with pytest.raises(TypeError):
        gqa.prefill(q.float(), q, q)


@pytest.mark.parametrize("args,expect", [
    # q, k, v, k_scale, v_scale, seqlens, out, B, h, n_kv, d, scale
    ((A, A, A, A, A, A, A, 2, 4, 2, 128, 0.1), None),
    ((A, A, A, 0, A, A, A, 2, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),      # null k_scale
    ((A, A, A, A, A + 2, A, A, 2, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),  # misaligned v_scale
    ((A, BAD, A, A, A, A, A, 2, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, A, A, 2, 4, 3, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, A, A, 2, 4, 2, 128, -1.0), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, A, A, A, 2, 4, 2, 96, 0.1), _lib.GQA_ERR_UNSUPPORTED),
])
def test_decode_fp8_rejects(L, args, expect):
    if expect is None:
        return   # a valid call would launch; covered by the GPU tests
    assert gqa.gqa_decode_fp8(*args, None) == expect


@pytest.mark.parametrize("table,mb,ps,npg,expect", [
    (0, 4, 64, 10, _lib.GQA_ERR_INVALID_ARG),          # null block table
    (A + 2, 4, 64, 10, _lib.GQA_ERR_INVALID_ARG),      # misaligned block table
    (A, 0, 64, 10, _lib.GQA_ERR_INVALID_ARG),          # max_blocks = 0
    (A, 4, 64, 0, _lib.GQA_ERR_INVALID_ARG),           # no pages
    (A, 4, 48, 10, _lib.GQA_ERR_INVALID_ARG),          # not a power of two
    (A, 4, 8, 10, _lib.GQA_ERR_INVALID_ARG),           # below 16
    (A, 4, 131072, 10, _lib.GQA_ERR_INVALID_ARG),      # above 65536
    (A, 1 << 20, 65536, 10, _lib.GQA_ERR_INVALID_ARG),  # max_blocks * page_size overflows int32
])
def test_decode_paged_rejects(L, table, mb, ps, npg, expect):
    assert gqa.gqa_decode_paged(A, A, A, table, mb, ps, npg, A, A, 2, 4, 2, 128, 0.1, None) == expect
    assert gqa.gqa_decode_paged_fp8(A, A, A, A, A, table, mb, ps, npg, A, A, 2, 4, 2, 128, 0.1, None) == expect


def test_decode_paged_fp8_needs_scales(L):
    assert gqa.gqa_decode_paged_fp8(A, A, A, 0, A, A, 4, 64, 10, A, A, 2, 4, 2, 128, 0.1, None) == \
        _lib.GQA_ERR_INVALID_ARG


def test_binding_rejects_bad_cache_dtypes():
    import torch
    q = torch.zeros(2, 4, 64, dtype=torch.bfloat16)
    k = torch.zeros(8, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):       # bf16 codes for an 8-bit cache
        gqa.decode_fp8(q, k, k, None, None, None)


@pytest.mark.parametrize("args,expect", [
    # q, k_new, v_new, k_pages, v_pages, table, max_blocks, page_size, num_pages, past, out, B, S_q, h, n_kv, d, scale
    ((0, A, A, A, A, A, 4, 64, 10, A, A, 2, 8, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),      # null q
    ((A, A, A, A, A, A, 4, 64, 10, 0, A, 2, 8, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),      # null past_lens
    ((A, A, A, BAD, A, A, 4, 64, 10, A, A, 2, 8, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),    # misaligned pages
    ((A, A, A, A, A, A, 4, 48, 10, A, A, 2, 8, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),      # page size
    ((A, A, A, A, A, A, 1, 64, 10, A, A, 2, 65, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),     # chunk > table
    ((A, A, A, A, A, A, 4, 64, 10, A, A, 2, 8, 4, 3, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),      # h % n_kv
    ((A, A, A, A, A, A, 4, 64, 10, A, A, 2, 8, 4, 2, 128, -1.0), _lib.GQA_ERR_INVALID_ARG),     # scale
    ((A, A, A, A, A, A, 4, 64, 10, A, A, 2, 8, 4, 2, 80, 0.1), _lib.GQA_ERR_UNSUPPORTED),       # d_h
])
def test_prefill_paged_rejects(L, args, expect):
    assert gqa.gqa_prefill_paged(*args, None) == expect


@pytest.mark.parametrize("args,expect", [
    # q_absorbed, c_kv, seqlens, out, B, h, d_c, scale
    ((0, A, A, A, 2, 32, 512, 0.04), _lib.GQA_ERR_INVALID_ARG),
    ((A, BAD, A, A, 2, 32, 512, 0.04), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A + 1, A, 2, 32, 512, 0.04), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, 0, 32, 512, 0.04), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, 2, 0, 512, 0.04), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, 2, 32, 512, float("nan")), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, A, 2, 32, 256, 0.04), _lib.GQA_ERR_UNSUPPORTED),
])
def test_mla_decode_rejects(L, args, expect):
    assert gqa.gqa_mla_decode(*args, None) == expect


@pytest.mark.parametrize("rows,expect", [
    (-1, _lib.GQA_ERR_INVALID_ARG),                # negative row count
    ((1 << 31), _lib.GQA_ERR_INVALID_ARG),         # above INT32_MAX (tile coordinates are 32-bit)
])
def test_row_checked_entry_points_reject_bad_row_counts(L, rows, expect):
    assert gqa.gqa_decode_rows(A, A, A, rows, A, A, 2, 4, 2, 128, 0.1, None) == expect
    assert gqa.gqa_decode_fp8_rows(A, A, A, rows, A, A, A, A, 2, 4, 2, 128, 0.1, None) == expect
    assert gqa.gqa_mla_decode_rows(A, A, rows, A, A, 2, 32, 512, 0.04, None) == expect


@pytest.mark.parametrize("args,expect", [
    # the argument checks of the forms without a row count apply too
    ((0, A, A, 100, A, A, 2, 4, 2, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, 100, A, A, 2, 4, 3, 128, 0.1), _lib.GQA_ERR_INVALID_ARG),
    ((A, A, A, 100, A, A, 2, 4, 2, 32, 0.1), _lib.GQA_ERR_UNSUPPORTED),
])
def test_decode_rows_rejects(L, args, expect):
    assert gqa.gqa_decode_rows(*args, None) == expect


def test_wait_test_library_exports_everything():
    """libgqa_b200_waittest.so: every entry point of gqa.h plus the one of gqa_waittest.h."""
    from attention_gqa_decode_b200.build import WAITTEST_LIB
    build()
    text = open(os.path.join(ROOT, "include", "gqa_waittest.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    extra = re.findall(r"^\s*int\s+(gqa_\w+)\s*\(", text, flags=re.M)
    assert extra == ["gqa_test_set_stall"]
    W = _lib.load_library(WAITTEST_LIB)
    for name in declared_functions() + extra:
        assert isinstance(getattr(W, name), ctypes._CFuncPtr), name
    # the product library has no test hook
    with pytest.raises(AttributeError):
        getattr(gqa.lib(), "gqa_test_set_stall")


def test_decode_dispatch_rule_on_cpu():
    """decode()'s choice of the split path for mid-sized groups at d = 128 (the branches
    that need no device query)."""
    import torch
    from attention_gqa_decode_b200 import _lib as L
    q = torch.zeros(64, 32, 128)
    k = torch.zeros(64 * 8192, 1, 128)
    assert L.use_split(q, k)                               # MQA, 32 heads per KV head
    assert L.use_split(torch.zeros(4, 64, 128), torch.zeros(4 * 300, 1, 128))
    assert not L.use_split(torch.zeros(4, 64, 128), torch.zeros(4 * 100, 1, 128))   # too few rows per sequence
    assert L.use_split(torch.zeros(4, 96, 128), torch.zeros(4 * 300, 2, 128))   # 48 heads per KV head
    assert not L.use_split(torch.zeros(4, 30, 128), torch.zeros(4 * 300, 4, 128))  # h % n_kv != 0


@pytest.mark.parametrize("B,h,n_kv,d", [
    (0, 32, 1, 128), (70000, 32, 1, 128), (4, 30, 4, 128), (4, 32, 0, 128), (4, 32, 1, 96),
    (65535, 512, 512, 128),   # 33.5 M (KV head, sequence) segments: past the split decode's 2^24
], ids=str)
def test_split_workspace_bytes_is_zero_for_rejected_sizes(L, B, h, n_kv, d):
    """gqa_decode_split_workspace_bytes answers 0 exactly where gqa_decode_split refuses the sizes
    (these cases return before the device's SM count is looked up)."""
    assert L.gqa_decode_split_workspace_bytes(B, h, n_kv, d) == 0


@pytest.mark.parametrize("B,h,d_c,rows,want,want_ws", [
    (16, 32, 512, 16 * 4096, 0, 0),    # the warp-level kernel fills the SMs (32 groups x 8 splits)
    (8, 32, 512, 8 * 32768, 1, 2),     # 128 warp-level CTAs, long sequences
    (1, 32, 512, 20000, 1, 2),
    (1, 32, 512, 8191, 0, 2),          # under 8192 rows per sequence (2048 with a workspace)
    (1, 32, 512, 2047, 0, 0),
    (1, 16, 512, 100000, 0, 0),        # 16 heads: one warp-level group is as wide
    (4, 64, 512, 4 * 16384, 1, 2),
    (5, 64, 512, 5 * 16384, 0, 0),     # 20 groups x 8 splits = 160 warp-level CTAs
    (8, 32, 512, 8 * 2048, 0, 2),      # 2048 rows per sequence are enough with a workspace
    (0, 32, 512, 0, -1, -1), (1, 0, 512, 10, -1, -1), (1, 32, 256, 10, -1, -1), (1, 32, 512, -1, -1, -1),
    (1, 32, 512, 2 ** 31, -1, -1),
], ids=str)
def test_mla_decode_path_rule(L, B, h, d_c, rows, want, want_ws):
    """gqa_mla_decode_path: the shape rules between the warp-level and the tensor-core MLA
    kernels as gqa.h states them, at the 148 SMs a B200 has (and the count assumed without one)."""
    assert L.gqa_mla_decode_path(B, h, d_c, rows, 0) == want
    assert L.gqa_mla_decode_path(B, h, d_c, rows, 1) == want_ws


@pytest.mark.parametrize("B,h,d_c,want", [
    (8, 32, 512, 8 * 18 * 65792),      # eighteen splits per sequence
    (1, 32, 512, 148 * 65792),         # one sequence over every SM
    (2, 80, 512, 6 * 24 * 65792),      # three 32-head groups
    (16, 32, 512, 0),                  # the warp-level kernel fills the SMs: never the tensor cores
    (300, 32, 512, 0), (4, 16, 512, 0),
    (0, 32, 512, 0), (70000, 32, 512, 0), (1, 0, 512, 0), (1, 32, 256, 0),
], ids=str)
def test_mla_split_workspace_bytes(L, B, h, d_c, want):
    assert L.gqa_mla_decode_split_workspace_bytes(B, h, d_c) == want


W256 = 1 << 20   # a 256-byte aligned stand-in workspace address (never dereferenced: these calls return first)


@pytest.mark.parametrize("args,ws,ws_bytes,expect", [
    # q_absorbed, c_kv, cache_rows, seqlens, out, B, h, d_c, scale
    ((0, A, 100, A, A, 2, 32, 512, 0.04), W256, 1 << 30, _lib.GQA_ERR_INVALID_ARG),
    ((A, A, 100, A + 1, A, 2, 32, 512, 0.04), W256, 1 << 30, _lib.GQA_ERR_INVALID_ARG),
    ((A, A, -1, A, A, 2, 32, 512, 0.04), W256, 1 << 30, _lib.GQA_ERR_INVALID_ARG),
    ((A, A, 100, A, A, 0, 32, 512, 0.04), W256, 1 << 30, _lib.GQA_ERR_INVALID_ARG),
    ((A, A, 100, A, A, 70000, 32, 512, 0.04), W256, 1 << 30, _lib.GQA_ERR_INVALID_ARG),
    ((A, A, 100, A, A, 2, 0, 512, 0.04), W256, 1 << 30, _lib.GQA_ERR_INVALID_ARG),
    ((A, A, 100, A, A, 2, 32, 512, -1.0), W256, 1 << 30, _lib.GQA_ERR_INVALID_ARG),
    ((A, A, 100, A, A, 2, 32, 256, 0.04), W256, 1 << 30, _lib.GQA_ERR_UNSUPPORTED),
    ((A, A, 100, A, A, 2, 32, 512, 0.04), 0, 1 << 30, _lib.GQA_ERR_INVALID_ARG),            # no workspace
    ((A, A, 100, A, A, 2, 32, 512, 0.04), W256 + 16, 1 << 30, _lib.GQA_ERR_INVALID_ARG),    # misaligned
    ((A, A, 20000, A, A, 2, 32, 512, 0.04), W256, 1000, _lib.GQA_ERR_INVALID_ARG),          # too small
])
def test_mla_decode_split_rejects(L, args, ws, ws_bytes, expect):
    """gqa_mla_decode_split's argument and workspace checks (all before any launch)."""
    assert gqa.gqa_mla_decode_split(*args, ws, ws_bytes, None) == expect
