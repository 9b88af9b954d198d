"""Algorithmic work counts used for the roofline figures.

KV bytes follow the cache-size formula of "Multi-query attention"
(pranaymahendrakar), section "Why this is a bandwidth argument, not a FLOP
argument": KV bytes = 2 * b * L * n_kv * d_h * S * B (b bytes per element,
L layers, n_kv KV heads, S context length, B batch).  The same count with
h in place of n_kv is the MHA cache of "Evolution of AI Attention
Mechanisms" (toolsku), "MHA Mathematical Formulation".

FLOP counts are the two contractions of exact attention, Q K^T and P V, at
2 flops per multiply-add; a causal prefill counts only the visible
(query, key) pairs.
"""
from __future__ import annotations


def kv_cache_bytes(b: int, L: int, n_kv: int, d_h: int, S: int, B: int) -> int:
    """2 * b * L * n_kv * d_h * S * B."""
    return 2 * b * L * n_kv * d_h * S * B


def decode_kv_bytes(seqlens, n_kv: int, d_h: int, elem_bytes: int = 2) -> int:
    """KV bytes one decode step must read: the formula with L=1, summed over ragged lengths."""
    return sum(kv_cache_bytes(elem_bytes, 1, n_kv, d_h, max(int(s), 0), 1) for s in seqlens)


def decode_flops(seqlens, h: int, d_h: int) -> int:
    """4 * h * d_h per cached token (Q K^T and P V), summed over the batch."""
    return sum(4 * h * d_h * max(int(s), 0) for s in seqlens)


def visible_pairs(S_q: int, S_kv: int, causal: bool) -> int:
    """(query, key) pairs a prefill evaluates; causal rows see keys j <= r + S_kv - S_q."""
    if not causal:
        return S_q * S_kv
    off = S_kv - S_q
    return sum(min(S_kv, r + off + 1) for r in range(S_q))


def prefill_flops(B: int, S_q: int, S_kv: int, h: int, d_h: int, causal: bool) -> int:
    return 4 * B * h * d_h * visible_pairs(S_q, S_kv, causal)


def chunk_prefill_flops(past_lens, S_q: int, h: int, d_h: int) -> int:
    """Causal chunk after past_lens[b] cached tokens: row r sees past + r + 1 keys;
    2 d_h flops for each of Q K^T and P V per (row, visible key, head)."""
    pairs = sum(max(int(p), 0) * S_q + S_q * (S_q + 1) // 2 for p in past_lens)
    return 4 * h * d_h * pairs


def prefill_io_bytes(B: int, S_q: int, S_kv: int, h: int, n_kv: int, d_h: int, elem_bytes: int = 2) -> int:
    """Compulsory HBM bytes: read Q, K, V once, write O once."""
    return elem_bytes * d_h * B * (2 * S_q * h + 2 * S_kv * n_kv)
