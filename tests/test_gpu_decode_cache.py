"""8-bit (E4M3) and paged decode caches: the CUDA path through the C ABI
against the fp64 oracle.

Tolerance as for the bf16 path (tests/_tol.py): max |GPU - oracle| <= 1e-2
below |oracle| = 4, the derived arithmetic bound above it (with f16 weights
for the 8-bit caches), and mean |GPU - oracle| <= 1e-3 per call.  The oracle
reads the same codes and scales,
so quantisation error is not part of the comparison: only the kernel's own
rounding (Q to f16, weights to f16, fp32 sums, bf16 output) is.
"""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import _lib, inputs

from tests._tol import MAX_ABS, MEAN_ABS, check  # noqa: F401

pytestmark = pytest.mark.gpu


def gpu_fp8(q, kc, vc, ks, vs, lens, scale=None):
    out = gqa.decode_fp8(q.cuda(), kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda(), lens.cuda(), scale=scale)
    torch.cuda.synchronize()
    return out.cpu()


def gpu_paged(q, kp, vp, bt, lens, ks=None, vs=None, scale=None):
    out = gqa.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), bt.cuda(), lens.cuda(), scale=scale,
                           k_scale=None if ks is None else ks.cuda(), v_scale=None if vs is None else vs.cuda())
    torch.cuda.synchronize()
    return out.cpu()


def status():
    return gqa.gqa_get_device_status()


# ----------------------------------------------------------------------------
# packed E4M3 caches

@pytest.mark.parametrize("B,h,n_kv,d,lens", [
    (3, 8, 2, 128, [1, 200, 1000]),
    (3, 8, 2, 64, [1, 200, 1000]),
    (5, 12, 4, 128, [1, 127, 128, 129, 255]),      # lengths around the 128-token stage
    (2, 32, 1, 128, [3000, 129]),                  # 32 heads per group
    (2, 64, 1, 128, [700, 5000]),                  # 64 heads per group
    (2, 64, 1, 64, [700, 5000]),
    (2, 128, 1, 128, [300, 2000]),                 # two 64-head slices
    (3, 8, 8, 128, [0, 300, 5]),                   # MHA, an empty sequence
    (1, 48, 4, 128, [10000]),                      # 12 heads per group, long
], ids=str)
def test_fp8_decode_parity(B, h, n_kv, d, lens):
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(40 + h + d, B, h, n_kv, d, lens)
    got = gpu_fp8(q, kc, vc, ks, vs, lens)
    check(got, oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs), "fp8 decode", v=vc,
          v_scale=vs, n_keys=int(lens.max()))
    for b in range(B):
        if int(lens[b]) <= 0:
            assert torch.all(got[b] == 0)
    assert status() == _lib.GQA_OK


@pytest.mark.parametrize("w", [inputs.GQA_DECODE_70B, inputs.MQA_DECODE_LONG, inputs.RAGGED_SWEEP[1]],
                         ids=lambda w: w.name)
def test_fp8_decode_workloads(w):
    """The decode workloads with their caches stored as E4M3, every output checked."""
    lens = inputs.ragged_lengths(w.seed, w.B, *w.ragged) if w.ragged else w.kv_len
    seed = w.seed * 1000 + w.n_kv if w.ragged else w.seed
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(seed, w.B, w.h, w.n_kv, w.d, lens)
    got = gpu_fp8(q, kc, vc, ks, vs, lens)
    check(got, oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs), w.name + " fp8", v=vc,
          v_scale=vs, n_keys=int(lens.max()))


def test_fp8_single_token_is_exact():
    # power-of-two V scales: code * scale is exact in fp32 and in bf16
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(3, 4, 16, 4, 128, 1)
    vs = torch.tensor([0.5, 2.0, 0.125, 1.0])
    got = gpu_fp8(q, kc, vc, ks, vs, lens)
    want = (vc.view(torch.float8_e4m3fn).float() * vs[None, :, None]).to(torch.bfloat16)
    for i in range(16):
        assert torch.equal(got[:, i], want[:, i // 4]), i


def test_fp8_group_mapping_bit_exact():
    B, h, n_kv, d = 2, 32, 4, 128
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(6, B, h, n_kv, d, [300, 77])
    codes = torch.tensor([float(g + 1) for g in range(n_kv)]).to(torch.float8_e4m3fn).view(torch.uint8)
    vc = codes[None, :, None].expand_as(vc).contiguous()
    got = gpu_fp8(q, kc, vc, ks, torch.ones(n_kv), lens)
    for i in range(h):
        assert torch.all(got[:, i].float() == float(i // (h // n_kv) + 1)), i


def test_fp8_scale_algebra_is_exact():
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(12, 4, 32, 8, 128, [100, 1000, 2000, 64])
    base = gpu_fp8(q, kc, vc, ks, vs, lens, scale=0.1)
    assert torch.equal(gpu_fp8(q, kc, vc, ks, vs * 2, lens, scale=0.1), base * 2)     # V scale: output x2
    assert torch.equal(gpu_fp8(q, kc, vc, ks * 2, vs, lens, scale=0.1),
                       gpu_fp8(q, kc, vc, ks, vs, lens, scale=0.2))                     # K scale: scores x2


def test_fp8_nan_code_stays_in_its_channel():
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(13, 2, 8, 2, 128, [50, 50])
    vc = vc.clone()
    vc[10, 1, 7] = 0x7F                                 # sequence 0, KV head 1, channel 7
    got = gpu_fp8(q, kc, vc, ks, vs, lens).float()
    ref = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs)
    assert torch.isnan(got[0, 4:8, 7]).all()
    assert np.isnan(ref[0, 4:8, 7]).all()
    mask = torch.ones_like(got, dtype=torch.bool)
    mask[0, 4:8, 7] = False
    assert torch.isfinite(got[mask]).all()
    assert float(np.abs(got.double().numpy()[mask.numpy()] - ref[mask.numpy()]).max()) <= MAX_ABS


def test_fp8_bad_scale_is_reported():
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(14, 2, 8, 2, 128, [50, 50])
    assert status() == _lib.GQA_OK
    gpu_fp8(q, kc, vc, torch.tensor([1.0, -1.0]), vs, lens)
    assert status() == _lib.GQA_ERR_INVALID_ARG
    gpu_fp8(q, kc, vc, ks, torch.tensor([float("nan"), 1.0]), lens)
    assert status() == _lib.GQA_ERR_INVALID_ARG
    assert status() == _lib.GQA_OK                      # reading clears it


# ----------------------------------------------------------------------------
# paged caches

@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_paged_parity(fp8, page_size):
    lens = [1, 100, 1000, 3333, 0, 257]
    B, h, n_kv, d = len(lens), 16, 2, 128
    if fp8:
        q, k, v, ks, vs, lens = inputs.decode_fp8_inputs(50 + page_size, B, h, n_kv, d, lens)
    else:
        q, k, v, lens = inputs.decode_inputs(50 + page_size, B, h, n_kv, d, lens)
        ks = vs = None
    kp, vp, bt = inputs.page_caches(60 + page_size, k, v, lens, page_size, spare_pages=5)
    got = gpu_paged(q, kp, vp, bt, lens, ks, vs)
    ref = oracle.decode_general(q, kp, vp, lens, fp8=fp8, k_scale=ks, v_scale=vs, block_table=bt,
                                page_size=page_size)
    check(got, ref, f"paged {'e4m3' if fp8 else 'bf16'} page {page_size}", v=vp, v_scale=vs,
          n_keys=int(lens.max()))
    assert torch.all(got[4] == 0)
    assert status() == _lib.GQA_OK


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
@pytest.mark.parametrize("h,n_kv,d", [(64, 1, 128), (32, 1, 128), (8, 8, 64), (64, 8, 64)])
def test_paged_group_sizes(fp8, h, n_kv, d):
    lens = [2000, 33, 700]
    B = len(lens)
    if fp8:
        q, k, v, ks, vs, lens = inputs.decode_fp8_inputs(70 + h + d, B, h, n_kv, d, lens)
    else:
        q, k, v, lens = inputs.decode_inputs(70 + h + d, B, h, n_kv, d, lens)
        ks = vs = None
    kp, vp, bt = inputs.page_caches(80, k, v, lens, 32, spare_pages=2)
    got = gpu_paged(q, kp, vp, bt, lens, ks, vs)
    check(got, oracle.decode_general(q, kp, vp, lens, fp8=fp8, k_scale=ks, v_scale=vs, block_table=bt,
                                     page_size=32), "paged group sizes", v=vp, v_scale=vs, n_keys=int(lens.max()))


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
def test_paged_workload_gqa_decode(fp8):
    """The GQA decode workload (B16 h64 n_kv8 d128 L4096) in 64-token pages, every output checked."""
    w = inputs.GQA_DECODE_70B
    if fp8:
        q, k, v, ks, vs, lens = inputs.decode_fp8_inputs(w.seed, w.B, w.h, w.n_kv, w.d, w.kv_len)
    else:
        q, k, v, lens = inputs.workload_inputs(w)
        ks = vs = None
    kp, vp, bt = inputs.page_caches(2, k, v, lens, 64)
    got = gpu_paged(q, kp, vp, bt, lens, ks, vs)
    check(got, oracle.decode_general(q, k, v, lens, fp8=fp8, k_scale=ks, v_scale=vs), w.name + " paged", v=v,
          v_scale=vs, n_keys=int(lens.max()))


def test_paged_bad_page_id_is_reported():
    lens = torch.tensor([300, 200], dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(90, 2, 8, 2, 128, lens)
    kp, vp, bt = inputs.page_caches(91, k, v, lens, 64)
    assert status() == _lib.GQA_OK
    bad = bt.clone()
    bad[1, 2] = kp.shape[0] + 5                          # past the pages: read as zeros
    got = gpu_paged(q, kp, vp, bad, lens)
    assert status() == _lib.GQA_ERR_INVALID_ARG
    assert torch.isfinite(got.float()).all()
    bad = bt.clone()
    bad[0, 0] = -1
    gpu_paged(q, kp, vp, bad, lens)
    assert status() == _lib.GQA_ERR_INVALID_ARG
    # sequence 0 untouched by the bad entry of sequence 1 in the first call
    check(got[:1], oracle.decode_general(q[:1], kp, vp, lens[:1], block_table=bt[:1], page_size=64), "seq 0",
          v=vp, n_keys=300)


def test_paged_length_beyond_block_table_is_cut_and_reported():
    lens = torch.tensor([128, 64], dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(92, 2, 8, 2, 128, lens)
    kp, vp, bt = inputs.page_caches(93, k, v, lens, 64)      # max_blocks = 2
    long = torch.tensor([1000, 64], dtype=torch.int32)
    got = gpu_paged(q, kp, vp, bt, long)
    assert status() == _lib.GQA_ERR_INVALID_ARG
    check(got, oracle.decode_general(q, kp, vp, lens, block_table=bt, page_size=64), "cut length", v=vp,
          n_keys=128)


def test_device_status_clean_after_cache_tests():
    assert status() == _lib.GQA_OK
