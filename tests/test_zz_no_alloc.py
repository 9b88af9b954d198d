"""gqa_decode_split_noalloc: the split-KV decode for callers that may not allocate
device memory (a plug-in inside another framework's memory pool, a serving loop
that forbids allocation after start-up).  Its workspace is a fixed array inside
the library instead of the caller's.

Called through the C ABI, twice in a row on the same inputs, and each result is
compared with gqa_decode_split (the entry point with a caller-provided
workspace) under the bound every GPU test uses (tests/_tol.py).  The file is
named to be collected last, and works alone in a fresh process as well as after
the other tests (the first call on the device performs the array's address
lookup).
"""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
from attention_gqa_decode_b200 import _lib, inputs
from tests._tol import check

pytestmark = pytest.mark.gpu


def _noalloc(q, k, v, lens, out):
    B, h, d = q.shape
    n_kv = k.shape[1]
    return gqa.lib().gqa_decode_split_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), k.shape[0], lens.data_ptr(),
                                              out.data_ptr(), B, h, n_kv, d, d ** -0.5,
                                              torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("B,h,n_kv,d,lens", [
    (6, 64, 1, 128, [3000, 10, 700, 5000, 64, 1]),     # 64 heads per KV head: balanced, one token group
    (5, 32, 1, 128, [4000, 17, 900, 0, 2500]),         # 32: balanced, two token groups
    (4, 32, 2, 64, [129, 2000, 0, 333]),               # d 64: heads as the MMA rows
], ids=str)
def test_noalloc_matches_the_workspace_entry_point_twice(B, h, n_kv, d, lens):
    q, k, v, L = (t.cuda() for t in inputs.decode_inputs(41 + d, B, h, n_kv, d, lens))
    want = gqa.decode_split(q, k, v, L)
    torch.cuda.synchronize()
    ref = want.float().cpu().double().numpy()
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        assert _noalloc(q, k, v, L, out) == _lib.GQA_OK
        torch.cuda.synchronize()
        check(out, ref, f"noalloc call {call + 1}", v=v, n_keys=max(lens))
        assert gqa.gqa_get_device_status() == _lib.GQA_OK


def test_noalloc_rejects_sizes_beyond_its_array():
    # 4 KV heads x 64 sequences need more partial slots than the fixed array holds
    B, h, n_kv, d = 64, 64, 4, 128
    assert gqa.gqa_decode_split_workspace_bytes(B, h, n_kv, d) > 16 << 20
    q, k, v, L = (t.cuda() for t in inputs.decode_inputs(43, B, h, n_kv, d, 8))
    out = torch.zeros_like(q)
    assert _noalloc(q, k, v, L, out) == _lib.GQA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(out == 0)                     # nothing launched
    assert np.isfinite(out.float().cpu().numpy()).all()


def test_noalloc_rejects_a_balanced_shape_beyond_its_array():
    # 32 heads per KV head at d 128: 296 CTA slots + one per (KV head, sequence), 33 KB each
    B, h, n_kv, d = 256, 32, 1, 128
    assert gqa.gqa_decode_split_workspace_bytes(B, h, n_kv, d) > 16 << 20
    assert gqa.gqa_decode_split_workspace_bytes(200, h, n_kv, d) <= 16 << 20
    q, k, v, L = (t.cuda() for t in inputs.decode_inputs(44, B, h, n_kv, d, 8))
    out = torch.zeros_like(q)
    assert _noalloc(q, k, v, L, out) == _lib.GQA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(out == 0)
