"""Chunked prefill over a paged cache (append + attention) through the C ABI,
against the fp64 oracle.

Attention: the bound of every path (tests/_tol.py): max |GPU - oracle| <= 1e-2
below |oracle| = 4, the derived arithmetic bound above, and mean <= 1e-3.  The
append is index work: the pages after the call must equal the oracle's pages
bit for bit, untouched slots (NaN here) included.
"""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import _lib, inputs

from tests._tol import MAX_ABS, MEAN_ABS, check  # noqa: F401

pytestmark = pytest.mark.gpu


def run(q, kn, vn, kp, vp, bt, past, scale=None):
    """Returns (out, k_pages after, v_pages after) on the CPU."""
    kpd, vpd = kp.cuda(), vp.cuda()
    out = gqa.prefill_paged(q.cuda(), kn.cuda(), vn.cuda(), kpd, vpd, bt.cuda(), past.cuda(), scale=scale)
    torch.cuda.synchronize()
    return out.cpu(), kpd.cpu(), vpd.cpu()


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("B,S_q,past,h,n_kv,d,ps", [
    (2, 200, [0, 300], 8, 2, 128, 64),
    (3, 128, [1, 127, 129], 4, 1, 128, 16),
    (2, 1, [500, 1000], 16, 4, 128, 32),          # a one-token chunk
    (2, 300, [256, 128], 8, 8, 64, 128),          # MHA, d 64
    (1, 512, [3000], 32, 8, 128, 256),            # long past, 4 query tiles
    (2, 64, [0, 0], 8, 2, 128, 16),               # no past: plain causal prefill
    (2, 257, [64, 1], 12, 4, 128, 512),           # pages larger than a key tile
], ids=str)
def test_chunk_prefill_parity_and_append(B, S_q, past, h, n_kv, d, ps):
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(100 + S_q, B, S_q, past, h, n_kv, d, ps,
                                                              spare_pages=3)
    got, kp2, vp2 = run(q, kn, vn, kp, vp, bt, past)
    ref, rkp, rvp = oracle.prefill_paged(q, kn, vn, kp, vp, bt, past)
    check(got, ref, "chunked prefill", v=torch.cat([vn.flatten(), vp.flatten()]), n_keys=int(past.max()) + S_q)
    assert np.array_equal(bits(kp2), rkp), "K pages after the append differ from the oracle's"
    assert np.array_equal(bits(vp2), rvp), "V pages after the append differ from the oracle's"
    assert gqa.gqa_get_device_status() == _lib.GQA_OK


def test_chunks_equal_one_prefill():
    """A 1024-token sequence in four 256-token chunks gives the rows of one causal prefill."""
    B, S, h, n_kv, d, ps = 2, 1024, 16, 4, 128, 64
    q, kn, vn, kp, vp, bt, _ = inputs.chunk_prefill_inputs(7, B, S, [0, 0], h, n_kv, d, ps)
    whole = gqa.prefill(q.cuda(), kn.cuda(), vn.cuda(), causal=True).cpu()
    kpd, vpd, btd = kp.cuda(), vp.cuda(), bt.cuda()
    outs = []
    for c in range(4):
        sl = slice(256 * c, 256 * (c + 1))
        past = torch.full((B,), 256 * c, dtype=torch.int32).cuda()
        outs.append(gqa.prefill_paged(q[:, sl].contiguous().cuda(), kn[:, sl].contiguous().cuda(),
                                      vn[:, sl].contiguous().cuda(), kpd, vpd, btd, past).cpu())
    torch.cuda.synchronize()
    chunked = torch.cat(outs, dim=1)
    ref = oracle.prefill(q, kn, vn, causal=True)
    check(chunked, ref, "four chunks", v=vn, n_keys=S)
    check(whole, ref, "one prefill", v=vn, n_keys=S)


def test_workload_chunk_sampled():
    """The last 512-token chunk of 4096-token sequences (B4 h32 n_kv8 d128, 64-token
    pages), the configuration the bench times: sampled rows checked against the
    dense oracle over the gathered cache."""
    B, S_q, P, h, n_kv, d, ps = 4, 512, 3584, 32, 8, 128, 64
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(4, B, S_q, [P] * B, h, n_kv, d, ps)
    got, kp2, vp2 = run(q, kn, vn, kp, vp, bt, past)
    btn = bt.numpy()
    rng = np.random.default_rng(4)
    for b in range(B):
        idx = [btn[b, t // ps] * ps + t % ps for t in range(P + S_q)]
        kfull = kp2.reshape(-1, n_kv, d)[idx][None]
        vfull = vp2.reshape(-1, n_kv, d)[idx][None]
        rows = sorted(set([0, 1, 127, 128, 255, 256, 511] + list(rng.integers(0, S_q, 8))))
        sample = [(0, int(rng.integers(0, h)), int(r)) for r in rows]
        ref = oracle.prefill_rows(q[b:b + 1], kfull, vfull, sample, causal=True)
        g = torch.stack([got[b, r, i] for _, i, r in sample])
        check(g, ref, f"sequence {b}", v=vfull, n_keys=P + S_q)
        # the append of this sequence, bit for bit
        assert torch.equal(kfull[0, P:].view(torch.int16), kn[b].view(torch.int16))
        assert torch.equal(vfull[0, P:].view(torch.int16), vn[b].view(torch.int16))


def test_bad_page_is_reported():
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(9, 2, 100, [200, 50], 8, 2, 128, 64)
    assert gqa.gqa_get_device_status() == _lib.GQA_OK
    bad = bt.clone()
    bad[1, 0] = kp.shape[0] + 3
    got, _, _ = run(q, kn, vn, kp, vp, bad, past)
    assert gqa.gqa_get_device_status() == _lib.GQA_ERR_INVALID_ARG
    assert torch.isfinite(got.float()).all()
    # sequence 0 does not use the bad entry
    ref, _, _ = oracle.prefill_paged(q[:1], kn[:1], vn[:1], kp, vp, bt[:1], past[:1])
    check(got[:1], ref, "sequence 0", v=torch.cat([vn.flatten(), vp.flatten()]), n_keys=300)


def test_past_beyond_table_is_cut_and_reported():
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(10, 1, 64, [100], 8, 2, 128, 64)
    # the table covers 3 pages = 192 positions; past 1000 is cut to 192 - 64 = 128 (the
    # result then reads reserved, unwritten slots, so only the report is checked)
    _, kp2, _ = run(q, kn, vn, kp, vp, bt, torch.tensor([1000], dtype=torch.int32))
    assert gqa.gqa_get_device_status() == _lib.GQA_ERR_INVALID_ARG
    btn = bt.numpy()
    written = torch.stack([kp2[btn[0, t // 64], t % 64] for t in range(128, 192)])
    assert torch.equal(written.view(torch.int16), kn[0].view(torch.int16))
