"""Pins for the oracle's 8-bit (E4M3) and paged decode caches.

What fixes each value (none of them is the oracle itself):
  - the E4M3 code table is checked against torch's own float8_e4m3fn
    conversion for all 256 codes;
  - the attention over an 8-bit cache is checked against the brute-force
    restatement run on caches dequantised through torch (code value times
    the head's scale), so a scale applied to the wrong head, to the wrong
    tensor, or not at all fails;
  - the roles of the two scales follow from the algebra: doubling every K
    scale doubles every score (the same as doubling the softmax scale),
    doubling every V scale doubles the output, both exactly in fp64;
  - a paged cache holds the same rows as the packed one, so its result is
    the packed result bit for bit, whatever the page order, the page size,
    or what the unused slots hold (NaN here).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_gqa_decode_b200 import inputs
from tests import _brute


def dequant(codes: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """codes uint8 [T, n_kv, d] -> fp64 values, through torch's E4M3 cast."""
    return codes.view(torch.float8_e4m3fn).to(torch.float64) * scale.to(torch.float64)[None, :, None]


def test_e4m3_table_matches_torch():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        got, want = oracle.e4m3_value(c), float(ref[c])
        if math.isnan(want):
            assert math.isnan(got), c
        else:
            assert got == want, (c, got, want)
    assert oracle.e4m3_value(0x7E) == 448.0          # largest finite magnitude
    assert oracle.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal


@pytest.mark.parametrize("n_kv", [1, 2, 4])
def test_fp8_decode_matches_bruteforce(n_kv):
    lens = torch.tensor([3, 0, 5, 1], dtype=torch.int32)
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(21 + n_kv, 4, 4, n_kv, 3, lens)
    # scales that differ per head and between K and V
    ks = ks * torch.linspace(0.7, 1.9, n_kv)
    vs = vs * torch.linspace(2.3, 0.4, n_kv)
    got = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs, scale=0.6)
    ref = _brute.decode(q, dequant(kc, ks), dequant(vc, vs), lens, 0.6)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    assert np.all(got[1] == 0.0)


def test_fp8_scale_roles():
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(5, 2, 8, 2, 16, [7, 4])
    base = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs, scale=0.25)
    # K scale x2 == softmax scale x2 (every score doubles)
    k2 = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks * 2, v_scale=vs, scale=0.25)
    s2 = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs, scale=0.5)
    assert np.array_equal(k2, s2)
    assert not np.allclose(k2, base)
    # V scale x2 == output x2
    v2 = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs * 2, scale=0.25)
    assert np.array_equal(v2, 2 * base)


def test_fp8_single_token_is_the_scaled_code():
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(8, 3, 4, 2, 8, 1)
    got = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs)
    want = dequant(vc, vs).numpy()                     # [3 tokens, n_kv, d]
    for b in range(3):
        for i in range(4):
            assert np.array_equal(got[b, i], want[b, i // 2])


def test_fp8_with_power_of_two_scales_equals_bf16_cache():
    """Dequantised values with power-of-two scales are exact bf16 numbers, so
    the 8-bit cache and the bf16 cache holding those numbers give one result."""
    q, kc, vc, _, _, lens = inputs.decode_fp8_inputs(9, 2, 6, 3, 8, [5, 9])
    ks = torch.tensor([0.25, 2.0, 0.0625])
    vs = torch.tensor([4.0, 0.5, 1.0])
    kb = dequant(kc, ks).to(torch.bfloat16)
    vb = dequant(vc, vs).to(torch.bfloat16)
    assert torch.equal(kb.to(torch.float64), dequant(kc, ks))
    got = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs)
    assert np.array_equal(got, oracle.decode(q, kb, vb, lens))


@pytest.mark.parametrize("page_size", [1, 2, 3, 16])
@pytest.mark.parametrize("fp8", [False, True])
def test_paged_equals_packed(page_size, fp8):
    lens = torch.tensor([7, 0, 1, 33, 16], dtype=torch.int32)
    if fp8:
        q, k, v, ks, vs, lens = inputs.decode_fp8_inputs(31, 5, 4, 2, 8, lens)
    else:
        q, k, v, lens = inputs.decode_inputs(31, 5, 4, 2, 8, lens)
        ks = vs = None
    kp, vp, bt = inputs.page_caches(77, k, v, lens, page_size, spare_pages=3)
    packed = oracle.decode_general(q, k, v, lens, fp8=fp8, k_scale=ks, v_scale=vs)
    paged = oracle.decode_general(q, kp, vp, lens, fp8=fp8, k_scale=ks, v_scale=vs, block_table=bt,
                                  page_size=page_size)
    assert np.all(np.isfinite(paged))                 # the NaN slots are never read
    assert np.array_equal(paged, packed)


def test_page_caches_layout():
    """The generator's page layout, checked row by row against the packed cache."""
    lens = torch.tensor([5, 0, 9], dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(3, 3, 2, 1, 4, lens)
    kp, vp, bt = inputs.page_caches(4, k, v, lens, 4, spare_pages=2)
    assert kp.shape == (2 + 0 + 3 + 2, 4, 1, 4)
    row = 0
    for b, L in enumerate(lens.tolist()):
        for t in range(L):
            page = int(bt[b, t // 4])
            assert torch.equal(kp[page, t % 4].view(torch.int16), k[row + t].view(torch.int16))
            assert torch.equal(vp[page, t % 4].view(torch.int16), v[row + t].view(torch.int16))
        row += L
    assert int(bt[1, 0]) == -1
    used = sorted(int(x) for x in bt.flatten() if x >= 0)
    assert len(used) == len(set(used)) == 5


def test_paged_rejects_bad_page():
    lens = torch.tensor([5], dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(3, 1, 2, 1, 4, lens)
    kp, vp, bt = inputs.page_caches(4, k, v, lens, 4)
    bad = bt.clone()
    bad[0, 1] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.decode_general(q, kp, vp, lens, block_table=bad, page_size=4)
    with pytest.raises(ValueError):                    # a length beyond the block table
        oracle.decode_general(q, kp, vp, torch.tensor([9], dtype=torch.int32), block_table=bt, page_size=4)


def test_fp8_nan_code_propagates():
    q, kc, vc, ks, vs, lens = inputs.decode_fp8_inputs(2, 1, 2, 1, 4, [3])
    vc = vc.clone()
    vc[1, 0, 2] = 0x7F
    got = oracle.decode_general(q, kc, vc, lens, fp8=True, k_scale=ks, v_scale=vs)
    assert np.isnan(got[0, :, 2]).all() and np.isfinite(np.delete(got[0], 2, axis=1)).all()
