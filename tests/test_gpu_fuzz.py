"""Seeded random shapes for every entry point, each against the fp64 oracle.

The named workloads and the hand-picked edge cases live in the other GPU test
files; this one draws sizes the others do not (group counts, head counts,
lengths around stage and page boundaries, chunk sizes, pasts, page sizes) from
a fixed seed, so a failure reproduces.  Bound: tests/_tol.py.
"""
import numpy as np
import pytest
import torch

import attention_gqa_decode_b200 as gqa
import oracle
from attention_gqa_decode_b200 import _lib, inputs
from tests._tol import check

pytestmark = pytest.mark.gpu

SPECIAL = [0, 1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 255, 256, 257]


def lengths(rng, B, hi):
    return [int(rng.choice(SPECIAL)) if rng.random() < 0.4 else int(rng.integers(0, hi)) for _ in range(B)]


def heads(rng):
    G = int(rng.choice([1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 40, 64, 96, 128]))
    n_kv = int(rng.choice([1, 2, 4])) if G > 16 else int(rng.choice([1, 2, 4, 8]))
    return G * n_kv, n_kv


def cuda(*ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("case", range(40))
def test_decode_fuzz(case):
    rng = np.random.default_rng(1000 + case)
    B = int(rng.integers(1, 6))
    h, n_kv = heads(rng)
    d = int(rng.choice([64, 128]))
    lens = lengths(rng, B, 3000)
    fp8 = case % 2 == 1
    page = int(rng.choice([0, 16, 32, 64, 128, 256, 512]))
    what = f"decode B{B} h{h} n_kv{n_kv} d{d} lens{lens} fp8={fp8} page={page}"
    if fp8:
        q, k, v, ks, vs, L = inputs.decode_fp8_inputs(case, B, h, n_kv, d, lens)
    else:
        q, k, v, L = inputs.decode_inputs(case, B, h, n_kv, d, lens)
        ks = vs = None
    if page:
        kp, vp, bt = inputs.page_caches(case, k, v, L, page, spare_pages=int(rng.integers(0, 3)))
        ref = oracle.decode_general(q, kp, vp, L, fp8=fp8, k_scale=ks, v_scale=vs, block_table=bt, page_size=page)
        qd, kd, vd, btd, ld = cuda(q, kp, vp, bt, L)
        out = gqa.decode_paged(qd, kd, vd, btd, ld, k_scale=None if ks is None else ks.cuda(),
                               v_scale=None if vs is None else vs.cuda())
    elif fp8:
        ref = oracle.decode_general(q, k, v, L, fp8=True, k_scale=ks, v_scale=vs)
        out = gqa.decode_fp8(*cuda(q, k, v, ks, vs, L))
    else:
        ref = oracle.decode(q, k, v, L)
        out = gqa.decode(*cuda(q, k, v, L))
    torch.cuda.synchronize()
    check(out, ref, what, v=v, v_scale=vs, n_keys=max(lens))
    assert gqa.gqa_get_device_status() == _lib.GQA_OK, what


@pytest.mark.parametrize("case", range(16))
def test_prefill_fuzz(case):
    rng = np.random.default_rng(2000 + case)
    B = int(rng.integers(1, 4))
    n_kv = int(rng.choice([1, 2, 4, 8]))
    h = n_kv * int(rng.choice([1, 2])) if n_kv == 8 else n_kv * int(rng.choice([1, 2, 4]))
    d = int(rng.choice([64, 128]))
    causal = bool(rng.random() < 0.7)
    S_q = int(rng.choice(SPECIAL[1:])) if rng.random() < 0.3 else int(rng.integers(1, 500))
    S_kv = S_q + int(rng.integers(0, 300)) if causal else int(rng.integers(1, 700))
    what = f"prefill B{B} S_q{S_q} S_kv{S_kv} h{h} n_kv{n_kv} d{d} causal={causal}"
    q, k, v = inputs.prefill_inputs(case, B, S_q, S_kv, h, n_kv, d)
    out = gqa.prefill(*cuda(q, k, v), causal=causal)
    torch.cuda.synchronize()
    check(out, oracle.prefill(q, k, v, causal=causal), what, v=v, n_keys=S_kv)


@pytest.mark.parametrize("case", range(12))
def test_chunk_prefill_fuzz(case):
    rng = np.random.default_rng(3000 + case)
    B = int(rng.integers(1, 3))
    n_kv = int(rng.choice([1, 2, 4]))
    h = n_kv * int(rng.choice([1, 2, 4]))
    d = int(rng.choice([64, 128]))
    S_q = int(rng.choice(SPECIAL[1:])) if rng.random() < 0.3 else int(rng.integers(1, 300))
    past = lengths(rng, B, 1000)
    page = int(rng.choice([16, 32, 64, 128, 256, 512]))
    what = f"chunk B{B} S_q{S_q} past{past} h{h} n_kv{n_kv} d{d} page{page}"
    q, kn, vn, kp, vp, bt, P = inputs.chunk_prefill_inputs(case, B, S_q, past, h, n_kv, d, page, spare_pages=1)
    ref, rkp, rvp = oracle.prefill_paged(q, kn, vn, kp, vp, bt, P)
    kpd, vpd = kp.cuda(), vp.cuda()
    out = gqa.prefill_paged(q.cuda(), kn.cuda(), vn.cuda(), kpd, vpd, bt.cuda(), P.cuda())
    torch.cuda.synchronize()
    check(out, ref, what, v=torch.cat([vn.flatten(), vp.flatten()]), n_keys=max(past) + S_q)
    bits = lambda t: t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)   # noqa: E731
    assert np.array_equal(bits(kpd), rkp) and np.array_equal(bits(vpd), rvp), what + ": pages after the append"


@pytest.mark.parametrize("case", range(12))
def test_mla_fuzz(case):
    rng = np.random.default_rng(4000 + case)
    B = int(rng.integers(1, 5))
    h = int(rng.integers(1, 81))
    lens = lengths(rng, B, 3000)
    what = f"MLA B{B} h{h} lens{lens}"
    q, c, L = inputs.mla_decode_inputs(case, B, h, 512, lens)
    out = gqa.mla_decode(*cuda(q, c, L))
    torch.cuda.synchronize()
    check(out, oracle.mla_decode(q, c, L), what, v=c, n_keys=max(lens))
    assert gqa.gqa_get_device_status() == _lib.GQA_OK, what
