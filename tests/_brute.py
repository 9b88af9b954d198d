"""Brute-force restatement used to pin the oracle on tiny inputs.

It follows a different route from the oracle on purpose: K and V are first
repeated per group exactly as the "GQA Implementation" code of "Evolution of
AI Attention Mechanisms" (toolsku) does it (insert an axis, expand it to
n_rep, reshape to h heads), and then every query head runs plain multi-head
attention with scalar Python loops and math.exp, no max subtraction.
"""
import math

import numpy as np
import torch


def repeat_kv(x: np.ndarray, n_rep: int) -> np.ndarray:
    """x [B, g, S, d] -> [B, g * n_rep, S, d] by expand + reshape."""
    if n_rep == 1:
        return x
    B, g, S, d = x.shape
    return np.broadcast_to(x[:, :, None, :, :], (B, g, n_rep, S, d)).reshape(B, g * n_rep, S, d)


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def mha_rows(q, k, v, visible, scale):
    """q [R,d], k/v [S,d] fp64; row r sees keys j < visible[r]."""
    R, d = q.shape
    out = np.zeros((R, v.shape[1]))
    for r in range(R):
        n = visible[r]
        if n <= 0:
            continue
        w = [math.exp(sum(q[r, c] * k[j, c] for c in range(d)) * scale) for j in range(n)]
        z = sum(w)
        for j in range(n):
            out[r] += (w[j] / z) * v[j]
    return out


def prefill(q, k, v, causal, scale):
    """q [B,S_q,h,d], k/v [B,S_kv,n_kv,d] torch bf16 -> fp64 [B,S_q,h,d]."""
    qf, kf, vf = as_f64(q), as_f64(k), as_f64(v)
    B, S_q, h, d = qf.shape
    S_kv, n_kv = kf.shape[1], kf.shape[2]
    # to the page's (B, heads, S, d) layout, then repeat per group
    kr = repeat_kv(kf.transpose(0, 2, 1, 3), h // n_kv)
    vr = repeat_kv(vf.transpose(0, 2, 1, 3), h // n_kv)
    out = np.zeros((B, S_q, h, d))
    vis = [min(S_kv, r + (S_kv - S_q) + 1) if causal else S_kv for r in range(S_q)]
    for b in range(B):
        for i in range(h):
            out[b, :, i, :] = mha_rows(qf[b, :, i, :], kr[b, i], vr[b, i], vis, scale)
    return out


def decode(q, k_cache, v_cache, seqlens, scale):
    qf, kf, vf = as_f64(q), as_f64(k_cache), as_f64(v_cache)
    B, h, d = qf.shape
    n_kv = kf.shape[1]
    out = np.zeros((B, h, d))
    off = 0
    for b in range(B):
        L = int(seqlens[b])
        if L > 0:
            kb = repeat_kv(kf[off:off + L].transpose(1, 0, 2)[None], h // n_kv)[0]
            vb = repeat_kv(vf[off:off + L].transpose(1, 0, 2)[None], h // n_kv)[0]
            for i in range(h):
                out[b, i] = mha_rows(qf[b, i][None], kb[i], vb[i], [L], scale)[0]
            off += L
    return out
