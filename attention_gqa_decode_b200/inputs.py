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
