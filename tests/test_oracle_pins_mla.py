"""Pins for the oracle's absorbed multi-head latent attention (MLA) decode.

"Evolution of AI Attention Mechanisms" (toolsku), "Generation 3: MLA": K is the
up-projection of the latent, K = c W_k_up^T per head, and absorbing W_k_up into the
query gives the same scores, Q K^T = (Q W_k_up) c^T.  The weights then multiply
the latent c itself.  Pinned here:
  - brute force on tiny inputs through the expand/reshape route (one KV head whose
    keys and values are both c);
  - the absorption identity, exactly: with small-integer q, W and c every score is
    an integer, so attention over the explicit keys K = c W^T (values c) and the
    absorbed decode over c with q' = q W give identical fp64 results;
  - one cached token returns that latent row exactly;
  - the default scale is d_c ** -0.5 (the factor in that page's code);
  - two tokens: the logistic closed form of a two-way softmax;
  - the softmax is over a set (row order within a sequence does not matter) and
    sequences do not see one another's rows.
"""
import numpy as np
import torch

import oracle
from attention_gqa_decode_b200 import inputs
from tests import _brute


def test_mla_matches_bruteforce():
    lens = torch.tensor([4, 0, 7], dtype=torch.int32)
    q, c, lens = inputs.mla_decode_inputs(5, 3, 4, 6, lens)
    got = oracle.mla_decode(q, c, lens, scale=0.3)
    ref = _brute.decode(q, c[:, None, :], c[:, None, :], lens, 0.3)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    assert np.all(got[1] == 0.0)


def test_absorption_identity_is_exact():
    rng = np.random.default_rng(0)
    B, h, d_h, d_c, L = 2, 3, 6, 6, 5        # d_h = d_c: the explicit keys and the values share a width
    W = rng.integers(-2, 3, size=(h, d_h, d_c)).astype(np.float64)      # per-head K up-projection
    q = rng.integers(-2, 3, size=(B, h, d_h)).astype(np.float64)
    c = rng.integers(-3, 4, size=(B * L, d_c)).astype(np.float64)
    lens = torch.full((B,), L, dtype=torch.int32)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)   # noqa: E731  (small integers: exact)
    q_abs = np.einsum("bhd,hdc->bhc", q, W)                            # q' = q W_k_up
    absorbed = oracle.mla_decode(bf(q_abs), bf(c), lens, scale=0.1)
    for i in range(h):
        K = c @ W[i].T                                                  # explicit keys of head i
        explicit = oracle.decode(bf(q[:, i:i + 1, :]), bf(K[:, None, :]), bf(c[:, None, :]), lens, scale=0.1)
        assert np.array_equal(absorbed[:, i:i + 1, :], explicit)


def test_single_token_returns_the_latent():
    q, c, lens = inputs.mla_decode_inputs(2, 3, 8, 16, 1)
    got = oracle.mla_decode(q, c, lens)
    for b in range(3):
        for i in range(8):
            assert np.array_equal(got[b, i], c[b].double().numpy())


def test_default_scale_is_latent_dim():
    q, c, lens = inputs.mla_decode_inputs(3, 2, 4, 16, [5, 9])
    assert np.array_equal(oracle.mla_decode(q, c, lens), oracle.mla_decode(q, c, lens, scale=16 ** -0.5))


def test_two_tokens_follow_the_logistic_closed_form():
    """Two cached tokens: the weight of the first is the logistic function of the score
    difference, sigma((q'.c0 - q'.c1) * scale), and the output mixes the two latents."""
    q, c, lens = inputs.mla_decode_inputs(4, 1, 3, 8, 2)
    scale = 0.25
    got = oracle.mla_decode(q, c, lens, scale=scale)
    qd, cd = q.double().numpy()[0], c.double().numpy()
    for i in range(3):
        delta = (qd[i] @ cd[0] - qd[i] @ cd[1]) * scale
        w0 = 1.0 / (1.0 + np.exp(-delta))
        np.testing.assert_allclose(got[0, i], w0 * cd[0] + (1.0 - w0) * cd[1], rtol=0, atol=1e-12)


def test_token_order_does_not_matter():
    """The softmax runs over a set: permuting a sequence's cached rows leaves its output."""
    lens = torch.tensor([9, 5], dtype=torch.int32)
    q, c, lens = inputs.mla_decode_inputs(6, 2, 4, 16, lens)
    perm = torch.cat([torch.randperm(9, generator=torch.Generator().manual_seed(1)),
                      9 + torch.randperm(5, generator=torch.Generator().manual_seed(2))])
    np.testing.assert_allclose(oracle.mla_decode(q, c[perm], lens), oracle.mla_decode(q, c, lens), rtol=0, atol=1e-12)


def test_sequences_are_independent():
    """Each sequence's output depends only on its own rows: the batch equals each sequence alone."""
    lens = torch.tensor([3, 0, 6, 1], dtype=torch.int32)
    q, c, lens = inputs.mla_decode_inputs(7, 4, 2, 8, lens)
    got = oracle.mla_decode(q, c, lens)
    off = 0
    for b in range(4):
        n = int(lens[b])
        alone = oracle.mla_decode(q[b:b + 1], c[off:off + n], lens[b:b + 1])
        np.testing.assert_allclose(got[b:b + 1], alone, rtol=0, atol=1e-13)
        off += n
