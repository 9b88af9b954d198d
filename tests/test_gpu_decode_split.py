"""gqa_decode_split (the batch's tokens divided evenly among the SMs, partial results
merged through the workspace) against the fp64 oracle.  By group size it runs the
tokens-as-rows tcgen05 kernel (up to 16 heads, d = 128), the balanced warp-level kernel
(17 to 64 heads, d = 128; two token groups per m-tile up to 32 heads) or the heads-as-rows
tcgen05 kernel (d = 64; and above 64 heads, with 2 or 4 copies of small groups at d = 64).

The kernel cuts sequences at arbitrary token positions, so the cases aim at
the places a cut can fall: lengths around the 64-token stage, sequences
shorter than a CTA's share and much longer than it, many sequences per CTA,
empty sequences, group sizes from 1 to 192 heads (two 128-head slices), d 64
and 128.  Bound: tests/_tol.py.
"""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import _lib, inputs
from tests._tol import check

pytestmark = pytest.mark.gpu


def run(q, k, v, lens, scale=None):
    out = gqa.decode_split(q.cuda(), k.cuda(), v.cuda(), lens.cuda(), scale=scale)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("G", [1, 4, 8, 16, 17, 24, 32, 40, 48, 56, 64, 96, 128, 192])
@pytest.mark.parametrize("d", [64, 128])
def test_split_group_sizes(G, d):
    n_kv = 2
    lens = torch.tensor([0, 1, 63, 64, 65, 130, 1000, 17, 4097], dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(G * 11 + d, len(lens), G * n_kv, n_kv, d, lens)
    got = run(q, k, v, lens)
    check(got, oracle.decode(q, k, v, lens), f"split G={G} d={d}", v=v, n_keys=int(lens.max()))
    assert torch.all(got[0] == 0)
    assert gqa.gqa_get_device_status() == _lib.GQA_OK


@pytest.mark.parametrize("B,h,n_kv,d,lo,hi", [
    (300, 32, 1, 128, 0, 200),      # many short sequences: several per CTA
    (5, 64, 1, 128, 1, 40),         # fewer tokens than SMs x a stage
    (40, 16, 4, 64, 500, 3000),
    (3, 128, 1, 128, 20000, 30000),  # few long sequences over every CTA
], ids=str)
def test_split_ragged(B, h, n_kv, d, lo, hi):
    lens = inputs.ragged_lengths(B + h, B, lo, hi)
    q, k, v, lens = inputs.decode_inputs(B * 7 + h, B, h, n_kv, d, lens)
    check(run(q, k, v, lens), oracle.decode(q, k, v, lens), f"split ragged B{B} h{h}", v=v,
          n_keys=int(lens.max()))


def test_split_one_long_sequence():
    q, k, v, lens = inputs.decode_inputs(31, 1, 64, 1, 128, 131072)
    check(run(q, k, v, lens), oracle.decode(q, k, v, lens), "split L=131072", v=v, n_keys=131072)


@pytest.mark.parametrize("w", [inputs.MQA_DECODE_LONG] + list(inputs.RAGGED_SWEEP), ids=lambda w: w.name)
def test_split_workloads(w):
    """The decode workloads through the split kernel, every output checked."""
    q, k, v, lens = inputs.workload_inputs(w)
    check(run(q, k, v, lens), oracle.decode(q, k, v, lens), w.name + " split", v=v, n_keys=int(lens.max()))


def test_split_matches_the_cluster_kernel_and_repeats():
    q, k, v, lens = (t.cuda() for t in inputs.decode_inputs(32, 20, 64, 2, 128, [700] * 10 + [3000] * 10))
    a = gqa.decode_split(q, k, v, lens)
    b = gqa.decode_split(q, k, v, lens)              # the same workspace, reused
    c = gqa.gqa_decode_rows                          # the cluster kernel, through its own entry point
    ref = torch.empty_like(q)
    assert c(q.data_ptr(), k.data_ptr(), v.data_ptr(), k.shape[0], lens.data_ptr(), ref.data_ptr(), 20, 64, 2, 128,
             128 ** -0.5, torch.cuda.current_stream().cuda_stream) == _lib.GQA_OK
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert (a.float() - ref.float()).abs().max().item() <= 1e-2


def test_split_exact_properties():
    # one token returns its V row exactly; V = the KV head's index maps groups bit-exactly
    q, k, v, lens = inputs.decode_inputs(33, 6, 64, 2, 128, 1)
    got = run(q, k, v, lens)
    for b in range(6):
        for i in range(64):
            assert torch.equal(got[b, i], v[b, i // 32]), (b, i)
    q, k, v, lens = inputs.decode_inputs(34, 3, 96, 3, 128, [300, 5000, 64])
    vg = torch.arange(3, dtype=torch.float32).view(1, 3, 1).expand(v.shape[0], 3, 128).to(torch.bfloat16)
    got = run(q, k, vg.contiguous(), lens)
    want = torch.arange(96).div(32, rounding_mode="floor").float().view(1, 96, 1).expand(3, 96, 128)
    assert torch.equal(got.float(), want)
    # scale 0: the mean of V
    q, k, v, lens = inputs.decode_inputs(35, 2, 32, 1, 128, [900, 70])
    check(run(q, k, v, lens, scale=0.0), oracle.decode(q, k, v, lens, scale=0.0), "split scale 0", v=v,
          n_keys=900)


def test_split_nan_in_the_next_sequence_stays_there():
    # sequence 0 (30 tokens) ends inside a stage whose remaining rows are sequence 1's
    q, k, v, lens = inputs.decode_inputs(36, 2, 32, 1, 128, [30, 100])
    v = v.clone()
    v[30, 0, 5] = float("nan")                        # sequence 1's first token
    got = run(q, k, v, lens)
    assert torch.isfinite(got[0].float()).all()
    assert torch.isnan(got[1, :, 5].float()).all()
    check(got[:1], oracle.decode(q[:1], k[:30], v[:30], lens[:1]), "split before a NaN row", v=v[:30], n_keys=30)


def test_split_lengths_past_the_cache_rows_are_cut_and_reported():
    q, k, v, lens = inputs.decode_inputs(37, 3, 32, 1, 128, torch.tensor([600, 600, 50], dtype=torch.int32))
    k, v = k[:1000].contiguous(), v[:1000].contiguous()
    assert gqa.gqa_get_device_status() == _lib.GQA_OK
    got = run(q, k, v, lens)
    assert gqa.gqa_get_device_status() == _lib.GQA_ERR_INVALID_ARG
    cut = torch.tensor([600, 400, 0], dtype=torch.int32)
    check(got, oracle.decode(q, k, v, cut), "split cut", v=v, n_keys=600)
    assert torch.all(got[2] == 0)


def test_decode_dispatch():
    """decode() sends wide groups, and batches too small to fill the SMs with the cluster
    kernel's splits, to gqa_decode_split (bit-identical to calling it directly)."""
    G = _lib.SPLIT_MIN_GROUP
    q, k, v, lens = (t.cuda() for t in inputs.decode_inputs(38, 4, G, 1, 128, 2000))
    assert _lib.use_split(q, k)
    assert torch.equal(gqa.decode(q, k, v, lens), gqa.decode_split(q, k, v, lens))
    q, k, v, lens = (t.cuda() for t in inputs.decode_inputs(38, 2, 16, 2, 128, 3000))   # 4 units
    assert _lib.use_split(q, k)
    assert torch.equal(gqa.decode(q, k, v, lens), gqa.decode_split(q, k, v, lens))
    q, k, v, lens = (t.cuda() for t in inputs.decode_inputs(38, 16, 64, 8, 128, 300))   # the GQA shape
    assert not _lib.use_split(q, k)
    q, k, v, lens = (t.cuda() for t in inputs.decode_inputs(38, 64, 32, 1, 128, 600))   # MQA: the balanced kernel
    assert _lib.use_split(q, k)
    assert torch.equal(gqa.decode(q, k, v, lens), gqa.decode_split(q, k, v, lens))


def test_split_status_clean():
    assert gqa.gqa_get_device_status() == _lib.GQA_OK


def test_split_running_max_rescales():
    """Keys along head 0's query, growing every 128 tokens: head 0's running max jumps by
    more than 2^8 several times inside a CTA's share (the lazy rescale of both kernels)."""
    for h, n_kv, d in ((32, 1, 128), (64, 2, 64), (256, 1, 128)):
        q, k, v, lens = inputs.decode_inputs(39 + h, 3, h, n_kv, d, [2000, 700, 5000])
        k = k.float()
        off = 0
        for b in range(3):
            u = q[b, 0].float() / q[b, 0].float().norm()
            for j in range(1, min(8, int(lens[b]) // 128)):
                k[off + 128 * j + 5, 0] = u * (8.0 * j)
            off += int(lens[b])
        k = k.to(torch.bfloat16)
        check(run(q, k, v, lens), oracle.decode(q, k, v, lens), f"split rescales h{h} d{d}", v=v, n_keys=5000)
