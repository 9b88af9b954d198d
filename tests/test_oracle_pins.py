"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics.

Each test is chosen so that a plausible slip in the oracle (a dropped scale,
a wrong group index such as i % n_kv, a transposed operand, a causal mask
off by one or aligned top-left, a missing normalisation) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from attention_gqa_decode_b200 import inputs, metrics
from tests import _brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


# ----------------------------------------------------------------------------
# brute force on tiny inputs (a different route: repeat K/V, scalar loops)

@pytest.mark.parametrize("n_kv", [1, 2, 3, 6])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("S_q,S_kv", [(5, 5), (3, 7), (1, 4)])
def test_prefill_matches_bruteforce(n_kv, causal, S_q, S_kv):
    q, k, v = inputs.prefill_inputs(11 + n_kv, 2, S_q, S_kv, 6, n_kv, 4)
    scale = 0.7
    got = oracle.prefill(q, k, v, causal=causal, scale=scale)
    ref = _brute.prefill(q, k, v, causal, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n_kv", [1, 2, 4])
def test_decode_matches_bruteforce(n_kv):
    lens = torch.tensor([3, 0, 1, 6], dtype=torch.int32)
    q, k, v, lens = inputs.decode_inputs(7, 4, 4, n_kv, 3, lens)
    got = oracle.decode(q, k, v, lens, scale=0.5)
    ref = _brute.decode(q, k, v, lens, 0.5)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    assert np.all(got[1] == 0.0)          # a sequence with no cached token gives zeros


# ----------------------------------------------------------------------------
# invariants and closed forms

def test_softmax_rows_sum_to_one():
    q, k, v = inputs.prefill_inputs(3, 1, 9, 9, 4, 2, 8)
    for causal in (True, False):
        P = oracle.prefill_probs(q, k, v, 0, 3, causal=causal)
        assert np.all(np.abs(P.sum(axis=1) - 1.0) < 1e-12)
        assert np.all(P >= 0)
        if causal:                          # nothing above the diagonal
            assert np.all(np.triu(P, 1) == 0.0)


def test_two_keys_closed_form():
    """Two keys: O = v0 + (v1 - v0) * sigmoid(s1 - s0)."""
    q, k, v = inputs.prefill_inputs(5, 1, 1, 2, 1, 1, 8)
    scale = 0.9
    out = oracle.prefill(q, k, v, causal=False, scale=scale)[0, 0, 0]
    qf, kf, vf = (t.double().numpy() for t in (q, k, v))
    s0 = float(qf[0, 0, 0] @ kf[0, 0, 0]) * scale
    s1 = float(qf[0, 0, 0] @ kf[0, 1, 0]) * scale
    sig = 1.0 / (1.0 + math.exp(-(s1 - s0)))
    want = vf[0, 0, 0] + (vf[0, 1, 0] - vf[0, 0, 0]) * sig
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-14)


def test_single_key_returns_v_exactly():
    q, k, v, lens = inputs.decode_inputs(9, 3, 8, 2, 16, torch.tensor([1, 1, 1], dtype=torch.int32))
    out = oracle.decode(q, k, v, lens)
    for b in range(3):
        for i in range(8):
            assert np.array_equal(out[b, i], v[b, i // 4].double().numpy())
    # causal prefill: row 0 sees key 0 only
    q, k, v = inputs.prefill_inputs(9, 2, 6, 6, 4, 2, 16)
    out = oracle.prefill(q, k, v, causal=True)
    for b in range(2):
        for i in range(4):
            assert np.array_equal(out[b, 0, i], v[b, 0, i // 2].double().numpy())


def test_identical_keys_and_zero_scale_give_mean_of_v():
    q, k, v = inputs.prefill_inputs(13, 1, 5, 5, 2, 1, 8)
    k_same = k[:, :1].expand(-1, 5, -1, -1).contiguous()
    for kk, scale in ((k_same, 0.3), (k, 0.0)):
        out = oracle.prefill(q, kk, v, causal=True, scale=scale)
        vf = v.double().numpy()
        for r in range(5):
            np.testing.assert_allclose(out[0, r, 0], vf[0, :r + 1, 0].mean(axis=0), rtol=0, atol=1e-14)


def test_shift_invariance():
    """Adding the same vector u to every key adds q.u to a whole row of scores: O unchanged."""
    g = torch.Generator().manual_seed(0)
    q = bf(torch.randint(-3, 4, (1, 4, 2, 8), generator=g))
    k = bf(torch.randint(-3, 4, (1, 6, 1, 8), generator=g))
    v, u = bf(torch.randn(1, 6, 1, 8, generator=g)), torch.randint(-2, 3, (8,), generator=g)
    k2 = bf(k.float() + u.float())                 # small integers: exact in bf16
    assert torch.equal(k2.float() - k.float(), u.float().expand_as(k.float()))
    for causal in (True, False):
        a = oracle.prefill(q, k, v, causal=causal, scale=0.25)
        b = oracle.prefill(q, k2, v, causal=causal, scale=0.25)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_key_permutation_invariance_decode():
    q, k, v, lens = inputs.decode_inputs(21, 1, 4, 2, 8, 10)
    perm = torch.randperm(10, generator=torch.Generator().manual_seed(1))
    a = oracle.decode(q, k, v, lens)
    b = oracle.decode(q, k[perm].contiguous(), v[perm].contiguous(), lens)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    assert not np.allclose(a[0, 0], oracle.decode(q, k, v[perm].contiguous(), lens)[0, 0])


def test_group_mapping_is_contiguous():
    """V of KV head g is the constant g: query head i must output i // (h / n_kv).

    (The probabilities sum to 1 only up to fp64 rounding, hence the 1e-13.)
    """
    h, n_kv, d = 12, 4, 8
    q, k, v = inputs.prefill_inputs(4, 2, 5, 5, h, n_kv, d)
    vg = torch.arange(n_kv, dtype=torch.float32).view(1, 1, n_kv, 1).expand(2, 5, n_kv, d).to(torch.bfloat16)
    out = oracle.prefill(q, k, vg.contiguous(), causal=True)
    for i in range(h):
        assert np.all(np.abs(out[:, :, i, :] - i // (h // n_kv)) < 1e-13), i
    q, kc, vc, lens = inputs.decode_inputs(4, 2, h, n_kv, d, 7)
    vg = torch.arange(n_kv, dtype=torch.float32).view(1, n_kv, 1).expand(14, n_kv, d).to(torch.bfloat16)
    out = oracle.decode(q, kc, vg.contiguous(), lens)
    for i in range(h):
        assert np.all(np.abs(out[:, i, :] - i // (h // n_kv)) < 1e-13), i


@pytest.mark.parametrize("n_kv", [1, 2, 4])
def test_gqa_equals_mha_on_repeated_kv(n_kv):
    """The page's GQA layer is MHA on K/V repeated per group; n_kv = 1 is MQA."""
    h = 4
    q, k, v = inputs.prefill_inputs(8, 2, 6, 6, h, n_kv, 8)
    rep = lambda t: torch.from_numpy(np.ascontiguousarray(
        _brute.repeat_kv(t.view(torch.int16).numpy().transpose(0, 2, 1, 3), h // n_kv).transpose(0, 2, 1, 3))
    ).view(torch.bfloat16)
    a = oracle.prefill(q, k, v, causal=True)
    b = oracle.prefill(q, rep(k), rep(v), causal=True)
    assert np.array_equal(a, b)


def test_causal_row_equals_truncated_full_attention():
    q, k, v = inputs.prefill_inputs(17, 1, 4, 9, 2, 1, 8)
    off = 9 - 4
    out = oracle.prefill(q, k, v, causal=True)
    for r in range(4):
        n = r + off + 1                     # bottom-right: the new queries are the last rows
        ref = oracle.prefill(q[:, r:r + 1], k[:, :n], v[:, :n], causal=False)
        np.testing.assert_array_equal(out[:, r], ref[:, 0])


def test_prefill_last_row_equals_decode():
    B, S, h, n_kv, d = 2, 7, 4, 2, 8
    q, k, v = inputs.prefill_inputs(23, B, S, S, h, n_kv, d)
    pre = oracle.prefill(q, k, v, causal=True)
    dec = oracle.decode(q[:, -1].contiguous(), k.reshape(B * S, n_kv, d), v.reshape(B * S, n_kv, d),
                        torch.full((B,), S, dtype=torch.int32))
    np.testing.assert_allclose(pre[:, -1], dec, rtol=0, atol=1e-13)


def test_sampled_rows_equal_full():
    q, k, v = inputs.prefill_inputs(31, 2, 20, 20, 4, 2, 8)
    full = oracle.prefill(q, k, v, causal=True)
    sample = [(0, 0, 0), (1, 3, 19), (0, 2, 7), (1, 1, 11)]
    rows = oracle.prefill_rows(q, k, v, sample, causal=True)
    for t, (b, i, r) in enumerate(sample):
        assert np.array_equal(rows[t], full[b, r, i])


def test_oracle_rejects_bad_shapes():
    q, k, v = inputs.prefill_inputs(1, 1, 4, 4, 3, 2, 8)      # h % n_kv != 0
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v)


# ----------------------------------------------------------------------------
# the KV-byte formula against the numbers the pages print

def test_kv_bytes_worked_example():
    gold = json.load(open(os.path.join(GOLDEN, "kv_cache_worked_example.json")))
    e = gold["mha_70b_layer"]
    per_layer = metrics.kv_cache_bytes(e["b"], e["L"], e["n_kv_times_d_h"], 1, e["S"], e["B"])
    assert per_layer == e["bytes_per_layer"] == 128 * 2 ** 20
    assert metrics.kv_cache_bytes(e["b"], e["layers"], e["n_kv_times_d_h"], 1, e["S"], e["B"]) == e["bytes_total"]
    f = gold["cache_fraction_of_mha_h64"]
    for n_kv, pct in f["rows"]:
        ratio = metrics.kv_cache_bytes(2, 1, n_kv, 128, 4096, 1) / metrics.kv_cache_bytes(2, 1, f["h"], 128, 4096, 1)
        assert ratio * 100 == pct
    m = gold["cache_fraction_of_mha_h128"]
    r = metrics.kv_cache_bytes(2, 1, m["n_kv"], m["d_h"], 1, 1) / metrics.kv_cache_bytes(2, 1, m["h"], m["d_h"], 1, 1)
    assert r * 100 == m["percent"] and 1 / r == m["compression"]
    mq = gold["mqa_32_heads"]
    assert metrics.kv_cache_bytes(2, 1, mq["h"], 128, 1, 1) // metrics.kv_cache_bytes(2, 1, 1, 128, 1, 1) == mq["reduction"]


def test_workload_byte_counts():
    w = inputs.GQA_DECODE_70B
    assert metrics.decode_kv_bytes([w.kv_len] * w.B, w.n_kv, w.d) == 268435456
    w = inputs.MQA_DECODE_LONG
    assert metrics.decode_kv_bytes([w.kv_len] * w.B, w.n_kv, w.d) == 268435456
    w = inputs.GQA_CAUSAL_PREFILL
    assert metrics.prefill_flops(w.B, w.S_q, w.S_kv, w.h, w.d, True) == 549890031616
    # visible pairs by brute force on a tiny case
    assert metrics.visible_pairs(3, 5, True) == sum(1 for r in range(3) for j in range(5) if j <= r + 2)
