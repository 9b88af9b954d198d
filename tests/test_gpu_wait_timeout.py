"""Bounded waits that run out, on the GPU, without a fault or a hang.

Every wait inside the kernels (a consumer waiting for a tile, the MMA thread
waiting for operands, a producer waiting for a free ring slot) gives up after
a time limit, records GQA_ERR_TIMEOUT in the device status word, lets the
copies already issued land, frees its tensor memory and returns.  These tests
drive that path through libgqa_b200_waittest.so (the same sources built with
a one-millisecond limit and a stall word, include/gqa_waittest.h): with the
stall word set, every producer leaves its first stage unloaded, so the waits
on it run out.  Each test checks that

- the stalled call returns promptly and the status word reads GQA_ERR_TIMEOUT;
- the status word is then clean, and the context still works: the next call
  with the stall cleared gives exactly the result of the product library.
"""
import ctypes
import time

import pytest
import torch

import attention_gqa_decode_b200 as gqa
from attention_gqa_decode_b200 import _lib, inputs
from attention_gqa_decode_b200.build import WAITTEST_LIB, build

pytestmark = pytest.mark.gpu

PROMPT_S = 5.0   # far above the waits' 1 ms limit, far below a hang


@pytest.fixture(scope="module")
def W():
    build()
    h = _lib.load_library(WAITTEST_LIB)
    h.gqa_test_set_stall.argtypes = [ctypes.c_int]
    h.gqa_test_set_stall.restype = ctypes.c_int
    torch.cuda.synchronize()
    assert h.gqa_get_device_status(None) == _lib.GQA_OK
    yield h
    h.gqa_test_set_stall(0)


def stream():
    return torch.cuda.current_stream().cuda_stream


def stalled_then_clean(W, launch, out):
    """Run launch(W) with the stall word set, then cleared; return the clean result."""
    torch.cuda.synchronize()
    assert W.gqa_test_set_stall(1) == _lib.GQA_OK
    try:
        t0 = time.monotonic()
        assert launch(W) == _lib.GQA_OK
        status = W.gqa_get_device_status(stream())
        elapsed = time.monotonic() - t0
    finally:
        assert W.gqa_test_set_stall(0) == _lib.GQA_OK
    assert status == _lib.GQA_ERR_TIMEOUT, status
    assert elapsed < PROMPT_S, elapsed
    assert W.gqa_get_device_status(stream()) == _lib.GQA_OK          # read once, then clear
    out.zero_()
    assert launch(W) == _lib.GQA_OK
    assert W.gqa_get_device_status(stream()) == _lib.GQA_OK
    torch.cuda.synchronize()
    return out.clone()


@pytest.mark.parametrize("B,h,n_kv,d,lens", [
    (1, 16, 2, 128, [3000]),           # one sequence split over a cluster of CTAs
    (200, 8, 2, 128, [700] * 200),     # one CTA per (sequence, KV head): no cluster merge
    (3, 64, 1, 64, [10, 500, 2000]),   # 64 heads per group, d 64
], ids=str)
def test_decode_wait_runs_out(W, B, h, n_kv, d, lens):
    q, k, v, L = (t.cuda() for t in inputs.decode_inputs(21, B, h, n_kv, d, lens))
    out = torch.empty_like(q)
    launch = lambda lib: lib.gqa_decode_rows(q.data_ptr(), k.data_ptr(), v.data_ptr(), k.shape[0], L.data_ptr(),  # noqa
                                             out.data_ptr(), B, h, n_kv, d, d ** -0.5, stream())
    got = stalled_then_clean(W, launch, out)
    want = torch.empty_like(q)    # the product library's same entry point
    assert gqa.gqa_decode_rows(q.data_ptr(), k.data_ptr(), v.data_ptr(), k.shape[0], L.data_ptr(), want.data_ptr(),
                               B, h, n_kv, d, d ** -0.5, stream()) == _lib.GQA_OK
    torch.cuda.synchronize()
    assert torch.equal(got, want)


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
def test_paged_decode_wait_runs_out(W, fp8):
    lens = [300, 1000]
    if fp8:
        q, k, v, ks, vs, L = inputs.decode_fp8_inputs(22, 2, 16, 2, 128, lens)
        ks, vs = ks.cuda(), vs.cuda()
    else:
        q, k, v, L = inputs.decode_inputs(22, 2, 16, 2, 128, lens)
    kp, vp, bt = inputs.page_caches(23, k, v, L, 32)
    q, kp, vp, bt, L = (t.cuda() for t in (q, kp, vp, bt, L))
    out = torch.empty_like(q)
    np_, ps, mb = kp.shape[0], kp.shape[1], bt.shape[1]

    def launch(lib):
        if fp8:
            return lib.gqa_decode_paged_fp8(q.data_ptr(), kp.data_ptr(), vp.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                                            bt.data_ptr(), mb, ps, np_, L.data_ptr(), out.data_ptr(), 2, 16, 2, 128,
                                            128 ** -0.5, stream())
        return lib.gqa_decode_paged(q.data_ptr(), kp.data_ptr(), vp.data_ptr(), bt.data_ptr(), mb, ps, np_,
                                    L.data_ptr(), out.data_ptr(), 2, 16, 2, 128, 128 ** -0.5, stream())

    got = stalled_then_clean(W, launch, out)
    want = gqa.decode_paged(q, kp, vp, bt, L, k_scale=ks if fp8 else None, v_scale=vs if fp8 else None)
    assert torch.equal(got, want)


@pytest.mark.parametrize("S,causal", [(300, True), (128, False), (700, True)], ids=str)
def test_prefill_wait_runs_out(W, S, causal):
    B, h, n_kv, d = 2, 4, 2, 128
    q, k, v = (t.cuda() for t in inputs.prefill_inputs(24, B, S, S, h, n_kv, d))
    out = torch.empty_like(q)
    launch = lambda lib: lib.gqa_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),  # noqa: E731
                                         B, S, S, h, n_kv, d, int(causal), d ** -0.5, stream())
    got = stalled_then_clean(W, launch, out)
    assert torch.equal(got, gqa.prefill(q, k, v, causal=causal))


def test_chunk_prefill_wait_runs_out(W):
    B, S_q, h, n_kv, d, ps = 2, 100, 8, 2, 128, 32
    q, kn, vn, kp, vp, bt, past = (t.cuda() for t in inputs.chunk_prefill_inputs(25, B, S_q, [200, 0], h, n_kv, d,
                                                                                 ps))
    out = torch.empty_like(q)
    kp0, vp0 = kp.clone(), vp.clone()
    launch = lambda lib: lib.gqa_prefill_paged(  # noqa: E731
        q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kp.data_ptr(), vp.data_ptr(), bt.data_ptr(), bt.shape[1], ps,
        kp.shape[0], past.data_ptr(), out.data_ptr(), B, S_q, h, n_kv, d, d ** -0.5, stream())
    got = stalled_then_clean(W, launch, out)
    kp2, vp2 = kp0.clone(), vp0.clone()
    want = gqa.prefill_paged(q, kn, vn, kp2, vp2, bt, past)
    assert torch.equal(got, want)
    assert torch.equal(kp.view(torch.int16), kp2.view(torch.int16))
    assert torch.equal(vp.view(torch.int16), vp2.view(torch.int16))


def test_mla_wait_runs_out(W):
    q, c, L = (t.cuda() for t in inputs.mla_decode_inputs(26, 3, 32, 512, [100, 2000, 33]))
    out = torch.empty_like(q)
    launch = lambda lib: lib.gqa_mla_decode_rows(q.data_ptr(), c.data_ptr(), c.shape[0], L.data_ptr(),  # noqa: E731
                                                 out.data_ptr(), 3, 32, 512, 512 ** -0.5, stream())
    got = stalled_then_clean(W, launch, out)
    assert torch.equal(got, gqa.mla_decode(q, c, L))


def test_mla_tensor_core_wait_runs_out(W):
    q, c, L = (t.cuda() for t in inputs.mla_decode_inputs(28, 2, 32, 512, [20000, 300]))
    assert W.gqa_mla_decode_path(2, 32, 512, c.shape[0], 0) == 1
    out = torch.empty_like(q)
    launch = lambda lib: lib.gqa_mla_decode_rows(q.data_ptr(), c.data_ptr(), c.shape[0], L.data_ptr(),  # noqa: E731
                                                 out.data_ptr(), 2, 32, 512, 512 ** -0.5, stream())
    got = stalled_then_clean(W, launch, out)
    want = torch.empty_like(q)   # the product library through the same entry (mla_decode takes the workspace path)
    assert gqa.gqa_mla_decode_rows(q.data_ptr(), c.data_ptr(), c.shape[0], L.data_ptr(), want.data_ptr(), 2, 32, 512,
                                   512 ** -0.5, stream()) == _lib.GQA_OK
    torch.cuda.synchronize()
    assert torch.equal(got, want)


def test_mla_tensor_core_workspace_wait_runs_out(W):
    q, c, L = (t.cuda() for t in inputs.mla_decode_inputs(29, 2, 32, 512, [20000, 300]))
    assert W.gqa_mla_decode_path(2, 32, 512, c.shape[0], 1) == 2
    nbytes = W.gqa_mla_decode_split_workspace_bytes(2, 32, 512)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    launch = lambda lib: lib.gqa_mla_decode_split(q.data_ptr(), c.data_ptr(), c.shape[0], L.data_ptr(),  # noqa: E731
                                                  out.data_ptr(), 2, 32, 512, 512 ** -0.5, ws.data_ptr(), nbytes,
                                                  stream())
    got = stalled_then_clean(W, launch, out)
    assert torch.equal(got, gqa.mla_decode(q, c, L))


def test_product_library_status_clean():
    assert gqa.gqa_get_device_status() == _lib.GQA_OK


@pytest.mark.parametrize("B,h,n_kv,d", [(6, 64, 1, 128), (5, 32, 1, 128), (3, 128, 1, 128), (4, 32, 2, 64)], ids=str)
def test_split_decode_wait_runs_out(W, B, h, n_kv, d):
    """The split-KV kernels (balanced warp-level with one and two token groups,
    heads-as-rows at d = 128 and 64, and their merge): the stalled call times out, and
    the next call through the same workspace is exact."""
    q, k, v, L = (t.cuda() for t in inputs.decode_inputs(27, B, h, n_kv, d, [3000, 10, 700, 5000, 64, 1][:B]))
    out = torch.empty_like(q)
    nbytes = W.gqa_decode_split_workspace_bytes(B, h, n_kv, d)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    launch = lambda lib: lib.gqa_decode_split(q.data_ptr(), k.data_ptr(), v.data_ptr(), k.shape[0],  # noqa: E731
                                              L.data_ptr(), out.data_ptr(), B, h, n_kv, d, d ** -0.5,
                                              ws.data_ptr(), nbytes, stream())
    got = stalled_then_clean(W, launch, out)
    assert torch.equal(got, gqa.decode_split(q, k, v, L))
