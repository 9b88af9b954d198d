"""Pins for the oracle's chunked prefill over a paged cache (append + attention).

Fixed independently of that function:
  - after the append, gathering the pages gives the past rows followed by the
    chunk's rows, and every other slot is untouched (bit for bit);
  - the attention equals the dense oracle prefill over the concatenated K/V
    with S_kv = past + S_q (bottom-right causal), bit for bit, and the
    brute-force restatement on tiny inputs;
  - two chunks in a row give the rows of one prefill over the whole sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from attention_gqa_decode_b200 import inputs
from tests import _brute


def gather(pages_bits, bt, b, n, page_size):
    """Rows 0..n-1 of sequence b from pages (uint16 bits) -> [n, n_kv, d] uint16."""
    return np.stack([pages_bits[bt[b, t // page_size], t % page_size] for t in range(n)]) if n else \
        np.zeros((0,) + pages_bits.shape[2:], dtype=np.uint16)


def bf(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("page_size", [1, 4, 16])
def test_append_writes_exactly_the_chunk(page_size):
    past = [5, 0, 17]
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(3, 3, 6, past, 4, 2, 8, page_size, spare_pages=2)
    _, kp2, vp2 = oracle.prefill_paged(q, kn, vn, kp, vp, bt, past)
    kp0 = kp.view(torch.int16).numpy().view(np.uint16)
    vp0 = vp.view(torch.int16).numpy().view(np.uint16)
    kbits = kn.view(torch.int16).numpy().view(np.uint16)
    vbits = vn.view(torch.int16).numpy().view(np.uint16)
    btn = bt.numpy()
    written = np.zeros(kp0.shape[:2], dtype=bool)
    for b in range(3):
        P = int(past[b])
        assert np.array_equal(gather(kp2, btn, b, P, page_size), gather(kp0, btn, b, P, page_size))
        for t in range(6):
            pos = P + t
            pg, sl = btn[b, pos // page_size], pos % page_size
            assert np.array_equal(kp2[pg, sl], kbits[b, t]) and np.array_equal(vp2[pg, sl], vbits[b, t])
            written[pg, sl] = True
    assert np.array_equal(kp2[~written], kp0[~written]) and np.array_equal(vp2[~written], vp0[~written])


@pytest.mark.parametrize("past", [[0, 0], [3, 3], [9, 2], [16, 31]])
def test_attention_equals_dense_prefill(past):
    ps = 4
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(7, 2, 5, past, 6, 3, 8, ps)
    out, kp2, vp2 = oracle.prefill_paged(q, kn, vn, kp, vp, bt, past, scale=0.4)
    btn = bt.numpy()
    for b in range(2):
        P = int(past[b])
        kfull = bf(gather(kp2, btn, b, P + 5, ps))[None]
        vfull = bf(gather(vp2, btn, b, P + 5, ps))[None]
        dense = oracle.prefill(q[b:b + 1], kfull, vfull, causal=True, scale=0.4)
        assert np.array_equal(out[b:b + 1], dense)
        ref = _brute.prefill(q[b:b + 1], kfull, vfull, True, 0.4)
        np.testing.assert_allclose(out[b:b + 1], ref, rtol=0, atol=1e-12)


def test_two_chunks_equal_one_prefill():
    """Sequence of 12 tokens: chunk of 7 (no past) then chunk of 5 (past 7)."""
    ps, h, n_kv, d = 4, 4, 2, 8
    q, kn, vn, kp, vp, bt, _ = inputs.chunk_prefill_inputs(11, 1, 12, [0], h, n_kv, d, ps)
    whole = oracle.prefill(q, kn, vn, causal=True)
    o1, kp1, vp1 = oracle.prefill_paged(q[:, :7], kn[:, :7], vn[:, :7], kp, vp, bt, [0])
    o2, _, _ = oracle.prefill_paged(q[:, 7:], kn[:, 7:], vn[:, 7:], bf(kp1), bf(vp1), bt, [7])
    assert np.array_equal(np.concatenate([o1, o2], axis=1), whole)


def test_rejects_bad_pages():
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(3, 1, 4, [6], 2, 1, 4, 4)
    bad = bt.clone()
    bad[0, 1] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.prefill_paged(q, kn, vn, kp, vp, bad, past)
    with pytest.raises(ValueError):     # past + S_q beyond the block table
        oracle.prefill_paged(q, kn, vn, kp, vp, bt, torch.tensor([9], dtype=torch.int32))
