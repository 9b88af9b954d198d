"""The largest sizes the entry points accept, against the fp64 oracle (bound: tests/_tol.py).

- decode with B = 65535 sequences (the grid limit the ABI enforces), lengths 0..3;
- one 131072-token sequence (each of the cluster's splits streams 16384 tokens);
- a 16384-row causal prefill, checked on sampled rows;
- MHA decode with 128 KV heads;
- a paged decode whose block table holds 2048 pages per sequence.
"""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import _lib, inputs
from tests._tol import check

pytestmark = pytest.mark.gpu


def test_decode_max_batch():
    B, h, n_kv, d = 65535, 8, 2, 64
    g = torch.Generator().manual_seed(1)
    lens = torch.randint(0, 4, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    q, k, v, lens = inputs.decode_inputs(1, B, h, n_kv, d, lens)
    out = gqa.decode(q.cuda(), k.cuda(), v.cuda(), lens.cuda())
    torch.cuda.synchronize()
    check(out, oracle.decode(q, k, v, lens), "decode B=65535", v=v, n_keys=3)
    assert torch.all(out.cpu()[lens == 0] == 0)
    assert gqa.gqa_get_device_status() == _lib.GQA_OK


def test_decode_one_long_sequence():
    q, k, v, lens = inputs.decode_inputs(2, 1, 16, 2, 128, 131072)
    out = gqa.decode(q.cuda(), k.cuda(), v.cuda(), lens.cuda())
    torch.cuda.synchronize()
    check(out, oracle.decode(q, k, v, lens), "decode L=131072", v=v, n_keys=131072)


def test_prefill_long_sequence_sampled():
    B, S, h, n_kv, d = 1, 16384, 8, 2, 128
    q, k, v = inputs.prefill_inputs(3, B, S, S, h, n_kv, d)
    out = gqa.prefill(q.cuda(), k.cuda(), v.cuda(), causal=True).cpu()
    rng = np.random.default_rng(3)
    rows = [0, 1, 127, 128, 8191, 8192, 16255, 16256, 16383] + list(rng.integers(0, S, 12))
    sample = [(0, int(rng.integers(0, h)), int(r)) for r in rows]
    ref = oracle.prefill_rows(q, k, v, sample, causal=True)
    check(torch.stack([out[b, r, i] for b, i, r in sample]), ref, "prefill S=16384", v=v, n_keys=S)


def test_decode_mha_128_heads():
    q, k, v, lens = inputs.decode_inputs(4, 2, 128, 128, 128, [1000, 3])
    out = gqa.decode(q.cuda(), k.cuda(), v.cuda(), lens.cuda())
    torch.cuda.synchronize()
    check(out, oracle.decode(q, k, v, lens), "MHA 128 heads", v=v, n_keys=1000)


def test_paged_decode_long_block_table():
    lens = [32768, 100]
    q, k, v, L = inputs.decode_inputs(5, 2, 8, 1, 128, lens)
    kp, vp, bt = inputs.page_caches(5, k, v, L, 16)      # 2048 pages for the long sequence
    assert bt.shape[1] == 2048
    out = gqa.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), bt.cuda(), L.cuda())
    torch.cuda.synchronize()
    check(out, oracle.decode_general(q, kp, vp, L, block_table=bt, page_size=16), "paged 2048 pages", v=vp,
          n_keys=32768)
    assert gqa.gqa_get_device_status() == _lib.GQA_OK
