"""fp64 CPU oracle for grouped-query attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The CUDA library never calls
it, and it shares no code with the CUDA library: the arithmetic lives in
``gqa_oracle.c`` (plain C, fp64, full score matrix per (batch, head)); this
file only compiles it with gcc, loads it with ctypes and marshals arrays.

Every function here is pinned by ``tests/test_oracle_pins.py`` to facts the
pages and the mathematics fix (closed forms, invariants, a brute-force
restatement through the expand-then-reshape K/V repetition, the KV-cache
worked number).  The 8-bit and paged decode caches (:func:`decode_general`,
:func:`e4m3_value`) are pinned by ``tests/test_oracle_pins_cache.py``
(torch's own E4M3 table, the brute-force restatement on torch-dequantised
caches, the algebra of the two scales, paged == packed bit for bit).
Parity status: pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB = os.path.join(_HERE, "libgqa_oracle.so")
_lock = threading.Lock()
_lib = None

_u16p = ctypes.POINTER(ctypes.c_uint16)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_int = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the C oracle (plain gcc, IEEE fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_prefill.argtypes = [_u16p, _u16p, _u16p, _f64p] + [_int] * 7 + [ctypes.c_double, _int]
            lib.oracle_prefill_rows.argtypes = ([_u16p, _u16p, _u16p, _f64p] + [_int] * 7 +
                                                [ctypes.c_double, _i32p, _int, _int])
            lib.oracle_decode.argtypes = [_u16p, _u16p, _u16p, _i32p, _f64p] + [_int] * 4 + [ctypes.c_double, _int]
            lib.oracle_prefill_probs.argtypes = ([_u16p, _u16p, _u16p, _f64p] + [_int] * 7 +
                                                 [ctypes.c_double, _int, _int])
            lib.oracle_decode_general.argtypes = ([_u16p, ctypes.c_void_p, ctypes.c_void_p, _int, _f32p, _f32p,
                                                   _i32p, _i32p, _int, _int, _int, _f64p] + [_int] * 4 +
                                                  [ctypes.c_double, _int])
            lib.oracle_prefill_paged.argtypes = ([_u16p, _u16p, _u16p, _u16p, _u16p, _i32p, _int, _int, _int, _i32p,
                                                  _f64p] + [_int] * 5 + [ctypes.c_double, _int])
            lib.oracle_prefill_paged.restype = _int
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_value.restype = ctypes.c_double
            for f in (lib.oracle_prefill, lib.oracle_prefill_rows, lib.oracle_decode, lib.oracle_prefill_probs,
                      lib.oracle_decode_general):
                f.restype = _int
            _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 bit patterns from a torch bf16 tensor or a uint16 array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _p(a, t):
    return a.ctypes.data_as(t)


def prefill(q, k, v, causal: bool = True, scale: float | None = None, n_threads: int = 0) -> np.ndarray:
    """Exact attention for q [B,S_q,h,d], k/v [B,S_kv,n_kv,d]; returns fp64 [B,S_q,h,d]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, S_q, h, d = qb.shape
    _, S_kv, n_kv, _ = kb.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((B, S_q, h, d), dtype=np.float64)
    rc = _load().oracle_prefill(_p(qb, _u16p), _p(kb, _u16p), _p(vb, _u16p), _p(out, _f64p),
                                B, S_q, S_kv, h, n_kv, d, int(bool(causal)), float(scale), n_threads)
    if rc:
        raise ValueError("oracle_prefill rejected its arguments")
    return out


def prefill_rows(q, k, v, sample, causal: bool = True, scale: float | None = None,
                 n_threads: int = 0) -> np.ndarray:
    """Output rows for the (b, i, r) triplets in ``sample`` ([n,3] int); returns fp64 [n,d]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, S_q, h, d = qb.shape
    _, S_kv, n_kv, _ = kb.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    s = np.ascontiguousarray(np.asarray(sample, dtype=np.int32).reshape(-1, 3))
    out = np.empty((s.shape[0], d), dtype=np.float64)
    rc = _load().oracle_prefill_rows(_p(qb, _u16p), _p(kb, _u16p), _p(vb, _u16p), _p(out, _f64p),
                                     B, S_q, S_kv, h, n_kv, d, int(bool(causal)), float(scale),
                                     _p(s, _i32p), s.shape[0], n_threads)
    if rc:
        raise ValueError("oracle_prefill_rows rejected its arguments")
    return out


def decode(q, k_cache, v_cache, seqlens, scale: float | None = None, n_threads: int = 0) -> np.ndarray:
    """One decode step: q [B,h,d], packed caches [T,n_kv,d], seqlens [B]; returns fp64 [B,h,d]."""
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    B, h, d = qb.shape
    n_kv = kb.shape[1]
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(B))
    if int(np.clip(lens, 0, None).sum()) > kb.shape[0]:
        raise ValueError("seqlens exceed the cache rows")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((B, h, d), dtype=np.float64)
    rc = _load().oracle_decode(_p(qb, _u16p), _p(kb, _u16p), _p(vb, _u16p), _p(lens, _i32p),
                               _p(out, _f64p), B, h, n_kv, d, float(scale), n_threads)
    if rc:
        raise ValueError("oracle_decode rejected its arguments")
    return out


def prefill_probs(q, k, v, b: int, i: int, causal: bool = True, scale: float | None = None) -> np.ndarray:
    """The S_q x S_kv softmax matrix of unit (b, i)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, S_q, h, d = qb.shape
    _, S_kv, n_kv, _ = kb.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    probs = np.empty((S_q, S_kv), dtype=np.float64)
    rc = _load().oracle_prefill_probs(_p(qb, _u16p), _p(kb, _u16p), _p(vb, _u16p), _p(probs, _f64p),
                                      B, S_q, S_kv, h, n_kv, d, int(bool(causal)), float(scale), b, i)
    if rc:
        raise ValueError("oracle_prefill_probs rejected its arguments")
    return probs


# ----------------------------------------------------------------------------
# 8-bit (E4M3) and paged decode caches

def e4m3_value(code: int) -> float:
    """The real number an OCP E4M3 code (0..255) stands for (NaN for 0x7f / 0xff)."""
    return float(_load().oracle_e4m3_value(int(code) & 0xFF))


def _codes(x) -> np.ndarray:
    """E4M3 codes as a contiguous uint8 array (from uint8 / float8_e4m3fn tensors or arrays)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint8
        return np.ascontiguousarray(x)
    import torch
    if x.dtype == torch.float8_e4m3fn:
        x = x.view(torch.uint8)
    assert x.dtype == torch.uint8, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().numpy())


def _f32(x, n: int) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x.cpu() if hasattr(x, "cpu") else x, dtype=np.float32).reshape(n))
    return a


def decode_general(q, k_cache, v_cache, seqlens, *, fp8: bool = False, k_scale=None, v_scale=None,
                   block_table=None, page_size: int = 0, scale: float | None = None,
                   n_threads: int = 0) -> np.ndarray:
    """One decode step over a bf16 or E4M3 cache, packed or paged; returns fp64 [B,h,d].

    Packed (``block_table is None``): caches [sum(seqlens), n_kv, d] as in :func:`decode`.
    Paged: caches [num_pages, page_size, n_kv, d]; ``block_table`` [B, max_blocks]
    int32; token t of sequence b sits in slot t % page_size of page
    block_table[b, t // page_size].  E4M3 caches take one fp32 scale per KV head
    for K (``k_scale``) and one for V (``v_scale``).
    """
    qb = _bits(q)
    B, h, d = qb.shape
    if fp8:
        kb, vb = _codes(k_cache), _codes(v_cache)
    else:
        kb, vb = _bits(k_cache), _bits(v_cache)
    n_kv = kb.shape[-2]
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(B))
    ks = _f32(k_scale, n_kv) if fp8 else None
    vs = _f32(v_scale, n_kv) if fp8 else None
    if block_table is None:
        if int(np.clip(lens, 0, None).sum()) > kb.shape[0]:
            raise ValueError("seqlens exceed the cache rows")
        bt, max_blocks, num_pages, page_size = None, 0, 0, 0
    else:
        bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32).reshape(B, -1))
        max_blocks, num_pages = bt.shape[1], kb.shape[0]
        if kb.shape[1] != page_size:
            raise ValueError("paged caches must be [num_pages, page_size, n_kv, d]")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((B, h, d), dtype=np.float64)
    rc = _load().oracle_decode_general(_p(qb, _u16p), kb.ctypes.data_as(ctypes.c_void_p),
                                       vb.ctypes.data_as(ctypes.c_void_p), int(bool(fp8)),
                                       _p(ks, _f32p) if fp8 else None, _p(vs, _f32p) if fp8 else None,
                                       _p(lens, _i32p), _p(bt, _i32p) if bt is not None else None,
                                       max_blocks, page_size, num_pages, _p(out, _f64p), B, h, n_kv, d,
                                       float(scale), n_threads)
    if rc:
        raise ValueError("oracle_decode_general rejected its arguments")
    return out


def prefill_paged(q, k_new, v_new, k_pages, v_pages, block_table, past_lens, scale: float | None = None):
    """Chunked causal prefill over a paged bf16 cache, with the append.

    q [B,S_q,h,d], k_new/v_new [B,S_q,n_kv,d], pages [num_pages,page_size,n_kv,d],
    block_table [B,max_blocks], past_lens [B].  Returns (out fp64 [B,S_q,h,d],
    k_pages_after, v_pages_after) -- the pages after the chunk's K/V were written
    at positions past_lens[b] .. past_lens[b] + S_q - 1 (as uint16 bf16 bits).
    """
    qb, kn, vn = _bits(q), _bits(k_new), _bits(v_new)
    kp, vp = _bits(k_pages).copy(), _bits(v_pages).copy()
    B, S_q, h, d = qb.shape
    n_kv = kn.shape[2]
    num_pages, page_size = kp.shape[0], kp.shape[1]
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32).reshape(B, -1))
    past = np.ascontiguousarray(np.asarray(past_lens, dtype=np.int32).reshape(B))
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((B, S_q, h, d), dtype=np.float64)
    rc = _load().oracle_prefill_paged(_p(qb, _u16p), _p(kn, _u16p), _p(vn, _u16p), _p(kp, _u16p), _p(vp, _u16p),
                                      _p(bt, _i32p), bt.shape[1], page_size, num_pages, _p(past, _i32p),
                                      _p(out, _f64p), B, S_q, h, n_kv, d, float(scale), 0)
    if rc:
        raise ValueError("oracle_prefill_paged rejected its arguments")
    return out, kp, vp


def mla_decode(q_absorbed, c_kv, seqlens, scale: float | None = None, n_threads: int = 0) -> np.ndarray:
    """Absorbed multi-head latent attention decode; returns fp64 [B,h,d_c].

    "Evolution of AI Attention Mechanisms" (toolsku), "Generation 3: MLA Multi-Head
    Latent Attention": the cache holds one shared latent c_kv per token; with the key
    up-projection absorbed into the query (q' = q W_k_up), the scores are
    q' c_kv^T * scale and the weights multiply c_kv itself.  So this is the plain
    decode of one KV head whose keys and values are both c_kv: q_absorbed
    [B,h,d_c], c_kv packed [sum(seqlens), d_c].  ``scale=None`` is d_c ** -0.5, the
    factor of that page's code.
    """
    cb = _bits(c_kv)
    d_c = cb.shape[-1]
    c3 = cb.reshape(-1, 1, d_c)
    if scale is None:
        scale = float(d_c) ** -0.5
    return decode_general(q_absorbed, c3, c3, seqlens, scale=scale, n_threads=n_threads)
