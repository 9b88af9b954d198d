"""Absorbed MLA decode through the C ABI against the fp64 oracle (bound: tests/_tol.py)."""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import _lib, inputs
from tests._tol import check

pytestmark = pytest.mark.gpu


def run(q, c, lens, scale=None):
    out = gqa.mla_decode(q.cuda(), c.cuda(), lens.cuda(), scale=scale)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("B,h,lens", [
    (3, 32, [1, 31, 33]),            # around the 32-token stage
    (2, 16, [1000, 5000]),
    (2, 128, [300, 2000]),           # eight 16-head groups
    (3, 40, [64, 0, 7]),             # a partial head group, an empty sequence
    (1, 32, [20000]),                # long: eight splits
], ids=str)
def test_mla_parity(B, h, lens):
    q, c, lens = inputs.mla_decode_inputs(60 + h, B, h, 512, lens)
    got = run(q, c, lens)
    check(got, oracle.mla_decode(q, c, lens), "MLA decode")
    for b in range(B):
        if int(lens[b]) <= 0:
            assert torch.all(got[b] == 0)
    assert gqa.gqa_get_device_status() == _lib.GQA_OK


def test_mla_workload():
    """B16 h32 d_c512 L4096, every output checked."""
    w = inputs.MLA_DECODE
    q, c, lens = inputs.mla_decode_inputs(w.seed, w.B, w.h, w.d, w.kv_len)
    check(run(q, c, lens), oracle.mla_decode(q, c, lens), w.name)


def test_mla_single_token_is_exact():
    q, c, lens = inputs.mla_decode_inputs(8, 4, 32, 512, 1)
    got = run(q, c, lens)
    for b in range(4):
        assert torch.equal(got[b], c[b][None].expand(32, -1)), b


def test_mla_default_scale():
    q, c, lens = inputs.mla_decode_inputs(9, 2, 16, 512, [100, 50])
    assert torch.equal(run(q, c, lens), run(q, c, lens, scale=512 ** -0.5))
