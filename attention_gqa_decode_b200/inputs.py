"""Seeded synthetic inputs shared by the CUDA path, the oracle, the tests and the bench.

This module holds no attention arithmetic: it only draws random numbers, casts
them to bf16 and names the workloads.  Both sides of every parity check read
the same bf16 bits produced here.

Recipe (one rule for every workload): a CPU ``torch.Generator`` seeded with
the workload's seed draws fp32 ``randn`` for q, then k, then v, each cast to
bf16 with round-to-nearest-even.  Ragged decode lengths are integers uniform
on a closed range, drawn by a generator seeded with the workload's seed; the
q/k/v of each point of the ragged sweep then come from a generator seeded
with ``seed * 1000 + n_kv``, so all points share one set of lengths.

8-bit caches are made from the same bf16 draws: per KV head, a scale
amax / 448 (the largest finite E4M3 magnitude) and codes from torch's own
cast of value / scale to ``float8_e4m3fn`` (round to nearest even).  Paged
caches hold the same rows as the packed ones, cut into pages of
``page_size`` tokens whose order in memory is a seeded random permutation;
the slots past a sequence's end, and the spare pages, are filled with NaN
(bf16 0x7fc0, E4M3 0x7f) so that reading them would show in any result.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One named workload: the shapes of a prefill or decode call."""

    name: str
    kind: str                 # "prefill" or "decode"
    seed: int
    B: int
    h: int
    n_kv: int
    d: int
    S_q: int = 0              # prefill only
    S_kv: int = 0             # prefill only
    causal: bool = True       # prefill only
    kv_len: int = 0           # decode, equal lengths
    ragged: tuple = ()        # decode, (lo, hi) closed range of lengths
    notes: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.h // self.n_kv


# The five workloads of the method's evaluation plan, by what they are.
TINY_MQA_PREFILL = Workload("tiny causal MQA prefill B1 S128 h4 n_kv1 d64", "prefill", 1,
                            B=1, h=4, n_kv=1, d=64, S_q=128, S_kv=128, causal=True)
GQA_DECODE_70B = Workload("GQA decode B16 h64 n_kv8 d128 L4096", "decode", 2,
                          B=16, h=64, n_kv=8, d=128, kv_len=4096)
MQA_DECODE_LONG = Workload("MQA decode B64 h32 n_kv1 d128 L8192", "decode", 3,
                           B=64, h=32, n_kv=1, d=128, kv_len=8192)
GQA_CAUSAL_PREFILL = Workload("GQA causal prefill B4 S4096 h32 n_kv8 d128", "prefill", 4,
                              B=4, h=32, n_kv=8, d=128, S_q=4096, S_kv=4096, causal=True)
RAGGED_SWEEP = tuple(
    Workload(f"ragged decode sweep B32 h64 d128 n_kv{n} L~U[512,8192]", "decode", 5,
             B=32, h=64, n_kv=n, d=128, ragged=(512, 8192))
    for n in (64, 8, 1)
)
ALL_WORKLOADS = (TINY_MQA_PREFILL, GQA_DECODE_70B, MQA_DECODE_LONG, GQA_CAUSAL_PREFILL) + RAGGED_SWEEP


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn_bf16(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def ragged_lengths(seed: int, B: int, lo: int, hi: int) -> torch.Tensor:
    """Integer lengths uniform on the closed range [lo, hi], int32, drawn first."""
    g = _gen(seed)
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def prefill_inputs(seed: int, B: int, S_q: int, S_kv: int, h: int, n_kv: int, d: int):
    """q [B,S_q,h,d], k and v [B,S_kv,n_kv,d], bf16 on the CPU."""
    g = _gen(seed)
    q = _randn_bf16(g, (B, S_q, h, d))
    k = _randn_bf16(g, (B, S_kv, n_kv, d))
    v = _randn_bf16(g, (B, S_kv, n_kv, d))
    return q, k, v


def decode_inputs(seed: int, B: int, h: int, n_kv: int, d: int, seqlens):
    """q [B,h,d]; packed caches [sum(seqlens), n_kv, d]; seqlens int32 [B].

    Sequence b's cached tokens start at row sum(seqlens[:b]) of each cache.
    ``seqlens`` may be an int (equal lengths) or a sequence of ints; a
    length <= 0 contributes no cache rows.
    """
    if isinstance(seqlens, int):
        seqlens = torch.full((B,), seqlens, dtype=torch.int32)
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).reshape(B)
    total = int(seqlens.clamp(min=0).sum())
    g = _gen(seed)
    q = _randn_bf16(g, (B, h, d))
    k = _randn_bf16(g, (total, n_kv, d))
    v = _randn_bf16(g, (total, n_kv, d))
    return q, k, v, seqlens


def workload_inputs(w: Workload):
    """Inputs for a named workload (CPU tensors)."""
    if w.kind == "prefill":
        return prefill_inputs(w.seed, w.B, w.S_q, w.S_kv, w.h, w.n_kv, w.d)
    if w.ragged:
        lens = ragged_lengths(w.seed, w.B, *w.ragged)
        # the same lengths for every n_kv of the sweep; q/k/v seeded per n_kv
        # from a generator of their own so they do not depend on the length draw
        return decode_inputs(w.seed * 1000 + w.n_kv, w.B, w.h, w.n_kv, w.d, lens)
    return decode_inputs(w.seed, w.B, w.h, w.n_kv, w.d, w.kv_len)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU tensor, as a contiguous uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


E4M3_MAX = 448.0          # largest finite magnitude of the OCP E4M3 format


def quantize_e4m3_per_head(x: torch.Tensor):
    """[T, n_kv, d] bf16 -> (codes uint8 [T, n_kv, d], scale float32 [n_kv]).

    scale[g] = amax over head g / 448 (1 for an all-zero head); codes are
    torch's round-to-nearest-even cast of x / scale[g] to float8_e4m3fn.
    """
    xf = x.to(torch.float32)
    amax = xf.abs().amax(dim=(0, 2)) if xf.shape[0] else torch.zeros(xf.shape[1])
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).to(torch.float32)
    codes = (xf / scale[None, :, None]).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes.view(torch.uint8), scale


def decode_fp8_inputs(seed: int, B: int, h: int, n_kv: int, d: int, seqlens):
    """The draws of :func:`decode_inputs`, with both caches stored as E4M3 codes.

    Returns q bf16 [B,h,d], k_codes and v_codes uint8 [sum(seqlens), n_kv, d],
    k_scale and v_scale float32 [n_kv], seqlens int32 [B].
    """
    q, k, v, seqlens = decode_inputs(seed, B, h, n_kv, d, seqlens)
    kc, ks = quantize_e4m3_per_head(k)
    vc, vs = quantize_e4m3_per_head(v)
    return q, kc, vc, ks, vs, seqlens


def page_caches(seed: int, k: torch.Tensor, v: torch.Tensor, seqlens, page_size: int, spare_pages: int = 0,
                reserve: int = 0):
    """Cut packed caches [sum(seqlens), n_kv, d] into pages.

    Returns (k_pages, v_pages [num_pages, page_size, n_kv, d], block_table
    int32 [B, max_blocks]).  Pages are placed in a seeded random order;
    block-table entries past a sequence's last page are -1; unused slots and
    the ``spare_pages`` extra pages hold NaN.  ``reserve`` extra tokens per
    sequence get pages too (left NaN), for a chunk to be appended.
    """
    lens = torch.as_tensor(seqlens, dtype=torch.int32).reshape(-1)
    B = lens.numel()
    n_blocks = [(max(int(L), 0) + reserve + page_size - 1) // page_size for L in lens.tolist()]
    max_blocks = max(1, max(n_blocks) if n_blocks else 1)
    num_pages = sum(n_blocks) + spare_pages
    g = _gen(seed)
    order = torch.randperm(max(num_pages, 1), generator=g)[:num_pages]
    T, n_kv, d = k.shape
    nan_code = 0x7FC0 if k.dtype == torch.bfloat16 else 0x7F
    raw = torch.int16 if k.dtype == torch.bfloat16 else torch.uint8
    fill = torch.tensor(nan_code, dtype=torch.int32).to(raw)
    kp = fill.repeat(max(num_pages, 1) * page_size * n_kv * d).view(max(num_pages, 1), page_size, n_kv, d)
    vp = kp.clone()
    bt = torch.full((B, max_blocks), -1, dtype=torch.int32)
    kr, vr = k.view(raw), v.view(raw)
    row, used = 0, 0
    for b in range(B):
        L = max(int(lens[b]), 0)
        for j in range(n_blocks[b]):
            page = int(order[used])
            used += 1
            n = max(0, min(page_size, L - j * page_size))
            kp[page, :n] = kr[row + j * page_size: row + j * page_size + n]
            vp[page, :n] = vr[row + j * page_size: row + j * page_size + n]
            bt[b, j] = page
        row += L
    return kp.view(k.dtype)[:num_pages], vp.view(v.dtype)[:num_pages], bt


def chunk_prefill_inputs(seed: int, B: int, S_q: int, past_lens, h: int, n_kv: int, d: int, page_size: int,
                         spare_pages: int = 0):
    """A chunk of S_q new tokens per sequence after past_lens[b] cached ones.

    Returns q [B,S_q,h,d], k_new and v_new [B,S_q,n_kv,d] (bf16), the paged
    caches holding the past tokens with pages reserved for the chunk (NaN
    until written), the block table, and past_lens int32 [B].  The past rows
    are drawn first (as a packed decode cache), then q, k_new, v_new.
    """
    past = torch.as_tensor(past_lens, dtype=torch.int32).reshape(B)
    g = _gen(seed)
    total = int(past.clamp(min=0).sum())
    k_past = _randn_bf16(g, (total, n_kv, d))
    v_past = _randn_bf16(g, (total, n_kv, d))
    q = _randn_bf16(g, (B, S_q, h, d))
    k_new = _randn_bf16(g, (B, S_q, n_kv, d))
    v_new = _randn_bf16(g, (B, S_q, n_kv, d))
    kp, vp, bt = page_caches(seed + 1, k_past, v_past, past, page_size, spare_pages=spare_pages, reserve=S_q)
    return q, k_new, v_new, kp, vp, bt, past


def mla_decode_inputs(seed: int, B: int, h: int, d_c: int, seqlens):
    """q_absorbed [B,h,d_c] and the packed latent cache c_kv [sum(seqlens), d_c], bf16.

    The absorbed query stands for q W_k_up of a trained model; with no weights here
    it is drawn directly, N(0,1) like the other inputs (cache first, then queries).
    """
    if isinstance(seqlens, int):
        seqlens = torch.full((B,), seqlens, dtype=torch.int32)
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).reshape(B)
    total = int(seqlens.clamp(min=0).sum())
    g = _gen(seed)
    c = _randn_bf16(g, (total, d_c))
    q = _randn_bf16(g, (B, h, d_c))
    return q, c, seqlens


MLA_DECODE = Workload("MLA absorbed decode B16 h32 d_c512 L4096", "decode", 6, B=16, h=32, n_kv=1, d=512,
                      kv_len=4096, notes="latent cache shared by all heads; K = V = c_kv")
MLA_DECODE_LONG = Workload("MLA absorbed decode B4 h32 d_c512 L65536", "decode", 7, B=4, h=32, n_kv=1, d=512,
                           kv_len=65536, notes="long sequences in a small batch (the tensor-core kernel's shapes)")
