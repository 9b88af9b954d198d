"""Absorbed MLA decode through the C ABI against the fp64 oracle (bound: tests/_tol.py)."""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import _lib, inputs
from tests._tol import check

pytestmark = pytest.mark.gpu


def run(q, c, lens, scale=None, entry="auto"):
    """entry "auto": mla_decode (gqa_mla_decode_split with a workspace where the path rule
    picks it, else gqa_mla_decode_rows); "rows": gqa_mla_decode_rows alone."""
    qd, cd, ld = q.cuda(), c.cuda(), lens.cuda()
    if entry == "auto":
        out = gqa.mla_decode(qd, cd, ld, scale=scale)
    else:
        B, h, d_c = q.shape
        out = torch.empty_like(qd)
        st = gqa.gqa_mla_decode_rows(qd.data_ptr(), cd.data_ptr(), cd.shape[0], ld.data_ptr(), out.data_ptr(), B, h,
                                     d_c, d_c ** -0.5 if scale is None else scale,
                                     torch.cuda.current_stream().cuda_stream)
        assert st == _lib.GQA_OK
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("B,h,lens", [
    (3, 32, [1, 31, 33]),
    (4, 32, [63, 64, 65, 129]),      # around 64 and 128 tokens
    (3, 8, [127, 128, 4097]),        # a partial head group; a ragged long sequence
    (2, 16, [1000, 5000]),
    (2, 128, [300, 2000]),           # several head groups
    (3, 40, [64, 0, 7]),             # a partial head group, an empty sequence
    (1, 32, [20000]),                # long: eight splits
    (1, 96, [9000]),                 # several head groups, several splits each
    # long sequences in small batches: the tensor-core kernel (asserted below)
    (2, 32, [0, 17000]),             # an empty sequence
    (3, 40, [9000, 255, 30000]),     # a partial 32-head group; a short sequence (remainder product)
    (4, 64, [8192, 1, 64, 40000]),   # one token; exactly one stage
    (16, 32, [4096] * 16),           # the workload's shape
], ids=str)
@pytest.mark.parametrize("entry", ["auto", "rows"])
def test_mla_parity(B, h, lens, entry):
    q, c, lens = inputs.mla_decode_inputs(60 + h, B, h, 512, lens)
    got = run(q, c, lens, entry=entry)
    check(got, oracle.mla_decode(q, c, lens), "MLA decode", v=c, n_keys=int(lens.max()))
    for b in range(B):
        if int(lens[b]) <= 0:
            assert torch.all(got[b] == 0)
    assert gqa.gqa_get_device_status() == _lib.GQA_OK


def test_mla_workload():
    """B16 h32 d_c512 L4096, every output checked."""
    w = inputs.MLA_DECODE
    q, c, lens = inputs.mla_decode_inputs(w.seed, w.B, w.h, w.d, w.kv_len)
    check(run(q, c, lens), oracle.mla_decode(q, c, lens), w.name, v=c, n_keys=w.kv_len)


def test_mla_single_token_is_exact():
    q, c, lens = inputs.mla_decode_inputs(8, 4, 32, 512, 1)
    got = run(q, c, lens)
    for b in range(4):
        assert torch.equal(got[b], c[b][None].expand(32, -1)), b


def test_mla_default_scale():
    q, c, lens = inputs.mla_decode_inputs(9, 2, 16, 512, [100, 50])
    assert torch.equal(run(q, c, lens), run(q, c, lens, scale=512 ** -0.5))


def test_mla_nan_in_previous_sequence_stays_there():
    # sequence 1 (30 tokens) is shorter than a stage: the box the kernel reads for it
    # ends at its last token and starts inside sequence 0, whose last row holds a NaN
    q, c, lens = inputs.mla_decode_inputs(10, 2, 32, 512, [100, 30])
    c = c.clone()
    c[99, 5] = float("nan")
    got = run(q, c, lens)
    assert torch.isnan(got[0].float()).any()
    check(got[1:], oracle.mla_decode(q[1:], c[100:], lens[1:]), "sequence after a NaN row", v=c[100:], n_keys=30)


def spiked_inputs(seed, B, h, lens):
    """Latent rows along head 0's query, growing every 64 tokens for five stages, so
    that head 0's running max jumps by more than 2^8 several times (the lazy rescale)."""
    q, c, L = inputs.mla_decode_inputs(seed, B, h, 512, lens)
    c = c.float()
    off = 0
    for b in range(B):
        u = q[b, 0].float() / q[b, 0].float().norm()
        for k in range(1, min(6, (int(L[b]) - 8) // 64 + 1)):
            c[off + 64 * k + 7] = u * (6.0 * k)
        off += int(L[b])
    return q, c.to(torch.bfloat16), L


def test_mla_running_max_rescale():
    q, c, lens = spiked_inputs(70, 3, 32, [1000, 300, 2049])
    check(run(q, c, lens), oracle.mla_decode(q, c, lens), "MLA with rescales", v=c, n_keys=2049)


def tc_path(B, h, lens, ws=0):
    return gqa.gqa_mla_decode_path(B, h, 512, int(sum(max(x, 0) for x in lens)), ws)


def test_mla_cases_cover_every_kernel():
    """The parity cases reach all three paths: the warp-level kernel, the tensor-core kernel
    with its splits merged in a cluster (gqa_mla_decode_rows) and through the workspace."""
    for B, h, lens in ((1, 32, [20000]), (1, 96, [9000]), (2, 32, [0, 17000]), (3, 40, [9000, 255, 30000]),
                       (4, 64, [8192, 1, 64, 40000])):
        assert tc_path(B, h, lens) == 1 and tc_path(B, h, lens, 1) == 2
    assert tc_path(16, 32, [4096] * 16) == 0 and tc_path(16, 32, [4096] * 16, 1) == 0
    assert tc_path(3, 32, [1, 31, 33]) == 0 and tc_path(3, 32, [1, 31, 33], 1) == 0


@pytest.mark.parametrize("entry", ["auto", "rows"])
def test_mla_tensor_core_single_token_is_exact(entry):
    q, c, lens = inputs.mla_decode_inputs(11, 2, 32, 512, [1, 20000])
    assert tc_path(2, 32, [1, 20000]) == 1 and tc_path(2, 32, [1, 20000], 1) == 2
    got = run(q, c, lens, entry=entry)
    assert torch.equal(got[0], c[0][None].expand(32, -1))


@pytest.mark.parametrize("entry", ["auto", "rows"])
def test_mla_tensor_core_nan_in_previous_sequence_stays_there(entry):
    # sequence 1 (30 tokens) is shorter than a 64-token stage: its box starts inside sequence 0
    q, c, lens = inputs.mla_decode_inputs(12, 2, 32, 512, [20000, 30])
    assert tc_path(2, 32, [20000, 30]) == 1 and tc_path(2, 32, [20000, 30], 1) == 2
    c = c.clone()
    c[19999, 5] = float("nan")
    got = run(q, c, lens, entry=entry)
    assert torch.isnan(got[0].float()).any()
    check(got[1:], oracle.mla_decode(q[1:], c[20000:], lens[1:]), "sequence after a NaN row", v=c[20000:], n_keys=30)


@pytest.mark.parametrize("entry", ["auto", "rows"])
def test_mla_tensor_core_running_max_rescale(entry):
    q, c, lens = spiked_inputs(71, 2, 32, [20000, 300])
    assert tc_path(2, 32, [20000, 300]) == 1 and tc_path(2, 32, [20000, 300], 1) == 2
    check(run(q, c, lens, entry=entry), oracle.mla_decode(q, c, lens), "MLA with rescales (tensor cores)", v=c,
          n_keys=20000)


def test_mla_split_rejects_a_small_workspace():
    q, c, lens = (t.cuda() for t in inputs.mla_decode_inputs(14, 2, 32, 512, [9000, 100]))
    need = gqa.gqa_mla_decode_split_workspace_bytes(2, 32, 512)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    args = (q.data_ptr(), c.data_ptr(), c.shape[0], lens.data_ptr(), out.data_ptr(), 2, 32, 512, 512 ** -0.5)
    s = torch.cuda.current_stream().cuda_stream
    assert gqa.gqa_mla_decode_split(*args, ws.data_ptr(), need - 1, s) == _lib.GQA_ERR_INVALID_ARG
    assert gqa.gqa_mla_decode_split(*args, ws.data_ptr() + 16, need - 16, s) == _lib.GQA_ERR_INVALID_ARG
    assert gqa.gqa_mla_decode_split(*args, None, need, s) == _lib.GQA_ERR_INVALID_ARG
    assert gqa.gqa_mla_decode_split(*args, ws.data_ptr(), need, s) == _lib.GQA_OK
    torch.cuda.synchronize()
    check(out.cpu(), oracle.mla_decode(*(t.cpu() for t in (q, c, lens))), "MLA split", v=c.cpu(), n_keys=9000)
