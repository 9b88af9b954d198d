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
  - the default scale is d_c ** -0.5 (the factor in that page's code).
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
