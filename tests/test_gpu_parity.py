"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Tolerance (bf16 inputs and outputs, fp32 accumulation): max |GPU - oracle|
<= 1e-2 and mean |GPU - oracle| <= 1e-3 per call, the oracle being unrounded
fp64; where |oracle| >= 4 (half a bf16 step is then above 1e-2) an element is
held to the bound the arithmetic allows instead (tests/_tol.py derives it).  Index and group-mapping work is checked
bit-exactly.
"""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import inputs

from tests._tol import MAX_ABS, MEAN_ABS, check  # noqa: F401

pytestmark = pytest.mark.gpu


def dev(*ts):
    return [t.cuda() for t in ts]


def gpu_decode(q, k, v, lens, scale=None):
    qd, kd, vd, ld = dev(q, k, v, lens)
    out = gqa.decode(qd, kd, vd, ld, scale=scale)
    torch.cuda.synchronize()
    return out.cpu()


def gpu_prefill(q, k, v, causal=True, scale=None):
    qd, kd, vd = dev(q, k, v)
    out = gqa.prefill(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return out.cpu()


# ----------------------------------------------------------------------------
# the named workloads

@pytest.mark.parametrize("w", [inputs.GQA_DECODE_70B, inputs.MQA_DECODE_LONG] + list(inputs.RAGGED_SWEEP),
                         ids=lambda w: w.name)
def test_decode_workload(w):
    q, k, v, lens = inputs.workload_inputs(w)
    check(gpu_decode(q, k, v, lens), oracle.decode(q, k, v, lens), w.name, v=v, n_keys=int(lens.max()))


def test_prefill_tiny_mqa():
    w = inputs.TINY_MQA_PREFILL
    q, k, v = inputs.workload_inputs(w)
    got = gpu_prefill(q, k, v, causal=True)
    check(got, oracle.prefill(q, k, v, causal=True), w.name, v=v, n_keys=w.S_kv)
    # row 0 attends to key 0 alone: exactly V[0] of its group
    for i in range(w.h):
        assert torch.equal(got[0, 0, i], v[0, 0, i // w.G]), i


def test_prefill_gqa_causal_sampled():
    """The full-size causal prefill, in the launch configuration the bench times,
    checked on sampled rows the oracle computes one by one."""
    w = inputs.GQA_CAUSAL_PREFILL
    q, k, v = inputs.workload_inputs(w)
    got = gpu_prefill(q, k, v, causal=True)
    rng = np.random.default_rng(4)
    rows = [0, 1, 127, 128, 129, 255, 256, 511, 2047, 2048, 4095] + list(rng.integers(0, w.S_q, 40))
    sample = [(int(rng.integers(0, w.B)), int(rng.integers(0, w.h)), int(r)) for r in rows]
    sample += [(w.B - 1, w.h - 1, w.S_q - 1), (0, 0, w.S_q - 1)]
    ref = oracle.prefill_rows(q, k, v, sample, causal=True)
    g = torch.stack([got[b, r, i] for b, i, r in sample])
    check(g, ref, w.name, v=v, n_keys=w.S_kv)
    assert torch.isfinite(got.float()).all()


# ----------------------------------------------------------------------------
# shapes: ragged tails, several tiles, bottom-right causal, d 64/128, the spectrum

@pytest.mark.parametrize("B,S_q,S_kv,h,n_kv,d,causal", [
    (1, 300, 300, 4, 2, 128, True),     # ragged tail over 3 key tiles
    (2, 200, 200, 6, 3, 64, False),
    (1, 100, 333, 8, 8, 128, True),     # MHA, bottom-right causal, S_q < S_kv
    (1, 257, 513, 4, 1, 64, True),      # MQA
    (1, 1, 1, 2, 1, 128, True),         # one query, one key
    (2, 129, 129, 3, 1, 128, True),
    (1, 384, 384, 2, 2, 64, False),
    (1, 640, 640, 2, 1, 128, True),     # several query-tile pairs
    (1, 64, 1000, 4, 2, 128, False),
])
def test_prefill_shapes(B, S_q, S_kv, h, n_kv, d, causal):
    q, k, v = inputs.prefill_inputs(100 + S_q, B, S_q, S_kv, h, n_kv, d)
    check(gpu_prefill(q, k, v, causal=causal), oracle.prefill(q, k, v, causal=causal), "prefill", v=v,
          n_keys=S_kv)


@pytest.mark.parametrize("G", [1, 3, 8, 12, 16, 24, 32, 48, 64, 128])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_group_sizes(G, d):
    n_kv = 2
    lens = torch.tensor([0, 1, 63, 64, 65, 130, 1000, 17], dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(G * 7 + d, len(lens), G * n_kv, n_kv, d, lens)
    got = gpu_decode(q, k, v, lens)
    check(got, oracle.decode(q, k, v, lens), f"decode G={G} d={d}", v=v, n_keys=int(lens.max()))
    assert torch.all(got[0] == 0)           # zero-length sequence -> zero row


# ----------------------------------------------------------------------------
# properties with exact answers

def test_single_key_is_exact():
    lens = torch.ones(5, dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(3, 5, 16, 4, 128, lens)
    got = gpu_decode(q, k, v, lens)
    for b in range(5):
        for i in range(16):
            assert torch.equal(got[b, i], v[b, i // 4]), (b, i)


def test_group_mapping_bit_exact():
    h, n_kv, d = 32, 8, 128
    q, k, v, lens = inputs.decode_inputs(5, 3, h, n_kv, d, 300)
    vg = torch.arange(n_kv, dtype=torch.float32).view(1, n_kv, 1).expand(v.shape[0], n_kv, d).to(torch.bfloat16)
    got = gpu_decode(q, k, vg.contiguous(), lens)
    want = torch.arange(h).div(h // n_kv, rounding_mode="floor").float().view(1, h, 1).expand(3, h, d)
    assert torch.equal(got.float(), want)
    qp, kp, vp = inputs.prefill_inputs(5, 1, 200, 200, h, n_kv, d)
    vg = torch.arange(n_kv, dtype=torch.float32).view(1, 1, n_kv, 1).expand(1, 200, n_kv, d).to(torch.bfloat16)
    got = gpu_prefill(qp, kp, vg.contiguous(), causal=True)
    want = torch.arange(h).div(h // n_kv, rounding_mode="floor").float().view(1, 1, h, 1).expand(1, 200, h, d)
    assert torch.equal(got.float(), want)


def test_zero_scale_is_mean_of_v():
    q, k, v, lens = inputs.decode_inputs(8, 2, 8, 2, 128, torch.tensor([700, 5], dtype=torch.int32))
    check(gpu_decode(q, k, v, lens, scale=0.0), oracle.decode(q, k, v, lens, scale=0.0), "scale 0 decode", v=v,
          n_keys=int(lens.max()))
    q, k, v = inputs.prefill_inputs(8, 1, 150, 150, 4, 2, 64)
    check(gpu_prefill(q, k, v, scale=0.0), oracle.prefill(q, k, v, scale=0.0), "scale 0 prefill", v=v, n_keys=150)


def test_large_scores_stay_finite():
    """Scores far from 0 exercise the running-max rescaling."""
    q, k, v = inputs.prefill_inputs(9, 1, 300, 300, 2, 1, 128)
    q = (q.float() * 4).to(torch.bfloat16)
    check(gpu_prefill(q, k, v, causal=True), oracle.prefill(q, k, v, causal=True), "large scores prefill", v=v,
          n_keys=300)
    q2, k2, v2, lens = inputs.decode_inputs(9, 2, 8, 1, 128, 900)
    q2 = (q2.float() * 4).to(torch.bfloat16)
    check(gpu_decode(q2, k2, v2, lens), oracle.decode(q2, k2, v2, lens), "large scores decode", v=v2, n_keys=900)


def test_split_count_does_not_change_the_result():
    """One sequence alone (split over many CTAs) and repeated through a large batch
    (cut at different points): equal up to fp32 rounding of the merge."""
    h, n_kv, d, L = 16, 2, 128, 3000
    q, k, v, lens = inputs.decode_inputs(12, 1, h, n_kv, d, L)
    alone = gpu_decode(q, k, v, lens)
    Bb = 200
    qb = q.expand(Bb, h, d).contiguous()
    kb = k.repeat(Bb, 1, 1)
    vb = v.repeat(Bb, 1, 1)
    batch = gpu_decode(qb, kb, vb, torch.full((Bb,), L, dtype=torch.int32))
    diff = (batch.float() - alone.float()).abs().max().item()
    assert diff <= 4e-3, diff


def test_gqa_equals_mha_on_repeated_kv():
    h, n_kv, d = 16, 4, 128
    q, k, v, lens = inputs.decode_inputs(13, 3, h, n_kv, d, torch.tensor([100, 2000, 777], dtype=torch.int32))
    rep = lambda t: t.repeat_interleave(h // n_kv, dim=1).contiguous()
    a = gpu_decode(q, k, v, lens)
    b = gpu_decode(q, rep(k), rep(v), lens)
    assert (a.float() - b.float()).abs().max().item() <= 4e-3


def test_prefill_last_row_matches_decode():
    B, S, h, n_kv, d = 2, 333, 8, 2, 128
    q, k, v = inputs.prefill_inputs(14, B, S, S, h, n_kv, d)
    pre = gpu_prefill(q, k, v, causal=True)
    dec = gpu_decode(q[:, -1].contiguous(), k.reshape(B * S, n_kv, d), v.reshape(B * S, n_kv, d),
                     torch.full((B,), S, dtype=torch.int32))
    assert (pre[:, -1].float() - dec.float()).abs().max().item() <= 1e-2


def test_repeatable():
    q, k, v, lens = inputs.workload_inputs(inputs.GQA_DECODE_70B)
    qd, kd, vd, ld = dev(q, k, v, lens)
    a = gqa.decode(qd, kd, vd, ld)
    b = gqa.decode(qd, kd, vd, ld)
    assert torch.equal(a, b)
    qp, kp, vp = dev(*inputs.prefill_inputs(1, 1, 512, 512, 8, 2, 128))
    assert torch.equal(gqa.prefill(qp, kp, vp), gqa.prefill(qp, kp, vp))


def test_device_status_clean():
    assert gqa.gqa_get_device_status() == 0


def test_lengths_past_the_cache_rows_are_cut_and_reported():
    """The binding passes the caches' row count (gqa_decode_rows): a sequence whose
    rows would run past the caches is cut to the rows that exist, reported, and
    nothing past the caches is read."""
    q, k, v, lens = inputs.decode_inputs(15, 3, 16, 2, 128, torch.tensor([600, 600, 50], dtype=torch.int32))
    k, v = k[:1000].contiguous(), v[:1000].contiguous()          # the caches hold 1000 of the 1250 rows
    assert gqa.gqa_get_device_status() == 0
    got = gpu_decode(q, k, v, lens)
    assert gqa.gqa_get_device_status() == 1                      # GQA_ERR_INVALID_ARG
    cut = torch.tensor([600, 400, 0], dtype=torch.int32)         # sequence 2 starts past the rows: empty
    check(got, oracle.decode(q, k, v, cut), "cut at the cache rows", v=v, n_keys=600)
    assert torch.all(got[2] == 0)
    # the same lengths over caches that hold every row: clean
    q, k, v, lens = inputs.decode_inputs(15, 3, 16, 2, 128, torch.tensor([600, 600, 50], dtype=torch.int32))
    gpu_decode(q, k, v, lens)
    assert gqa.gqa_get_device_status() == 0


def test_mla_and_fp8_lengths_past_the_cache_rows_are_cut_and_reported():
    q, c, lens = inputs.mla_decode_inputs(16, 2, 32, 512, [300, 300])
    c = c[:450].contiguous()
    got = gqa.mla_decode(q.cuda(), c.cuda(), lens.cuda()).cpu()
    assert gqa.gqa_get_device_status() == 1
    check(got, oracle.mla_decode(q, c, torch.tensor([300, 150], dtype=torch.int32)), "MLA cut", v=c, n_keys=300)
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(17, 2, 8, 2, 128, [300, 300])
    kc, vc = kc[:450].contiguous(), vc[:450].contiguous()
    got = gqa.decode_fp8(q.cuda(), kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda(), lens.cuda()).cpu()
    assert gqa.gqa_get_device_status() == 1
    ref = oracle.decode_general(q, kc, vc, torch.tensor([300, 150], dtype=torch.int32), fp8=True, k_scale=ks,
                                v_scale=vs)
    check(got, ref, "E4M3 cut", v=vc, v_scale=vs, n_keys=300)


def test_prefill_output_is_complete_for_work_queued_behind_it():
    """A causal prefill is two launches (the common query-tile pairs, then the pairs whose
    rows see few keys, started beside the first one's last wave).  Work queued behind the
    call on the same stream must see every output row: copy the output on that stream,
    before any host synchronisation, and compare the copy with the oracle."""
    B, S, h, n_kv, d = 2, 1024, 8, 2, 128
    q, k, v = inputs.prefill_inputs(61, B, S, S, h, n_kv, d)
    ref = oracle.prefill(q, k, v, causal=True)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        for _ in range(3):
            out = torch.full_like(qd, float("nan"))
            got = gqa.prefill(qd, kd, vd, causal=True, out=out)
            snap = got.clone()                     # queued on `side`, behind both launches
            side.synchronize()
            assert torch.isfinite(snap.float()).all()
            check(snap.cpu(), ref, "prefill output copied on the same stream", v=v, n_keys=S)
