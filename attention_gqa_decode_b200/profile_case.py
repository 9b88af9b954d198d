"""Run a named workload a few times on cuda:0, for profilers (ncu -k ... -s ... -c ...).

    python -m attention_gqa_decode_b200.profile_case decode GQA_DECODE_70B 3
    python -m attention_gqa_decode_b200.profile_case prefill GQA_CAUSAL_PREFILL 2
    python -m attention_gqa_decode_b200.profile_case decode RAGGED_SWEEP:2 3
    python -m attention_gqa_decode_b200.profile_case decode_fp8 GQA_DECODE_70B 3
    python -m attention_gqa_decode_b200.profile_case decode_paged64 GQA_DECODE_70B 3
    python -m attention_gqa_decode_b200.profile_case decode_paged64_fp8 GQA_DECODE_70B 3

    python -m attention_gqa_decode_b200.profile_case mla MLA_DECODE 3
    python -m attention_gqa_decode_b200.profile_case prefill_chunk GQA_CAUSAL_PREFILL 2

``decode_fp8`` stores the decode workload's caches as E4M3 codes (one scale
per KV head); ``decode_paged<N>`` cuts them into pages of N tokens, and a
``_fp8`` suffix does both.  ``prefill_chunk`` runs the last 512-token chunk of
the prefill workload's sequences (3584 past tokens in 64-token pages).

The inputs are the seeded synthetic ones; nothing is checked or timed here.
"""
from __future__ import annotations

import sys

import torch

import attention_gqa_decode_b200 as gqa
from attention_gqa_decode_b200 import inputs


def main(argv) -> int:
    kind, name = argv[0], argv[1]
    n = int(argv[2]) if len(argv) > 2 else 3
    if ":" in name:
        name, idx = name.split(":")
        w = getattr(inputs, name)[int(idx)]
    else:
        w = getattr(inputs, name)
    base = kind.split("_")[0]
    if kind == "mla":
        q, c, lens = (x.cuda() for x in inputs.mla_decode_inputs(w.seed, w.B, w.h, w.d, w.kv_len))
        for _ in range(n):
            gqa.mla_decode(q, c, lens)
        torch.cuda.synchronize()
        st = gqa.gqa_get_device_status()
        print(f"{w.name}: {n} calls, device status {st}")
        return 0 if st == 0 else 1
    if kind == "prefill_chunk":
        S_q, P = 512, w.S_q - 512
        t = inputs.chunk_prefill_inputs(w.seed, w.B, S_q, [P] * w.B, w.h, w.n_kv, w.d, 64)
        q, kn, vn, kp, vp, bt, past = (x.cuda() for x in t)
        for _ in range(n):
            gqa.prefill_paged(q, kn, vn, kp, vp, bt, past)
        torch.cuda.synchronize()
        st = gqa.gqa_get_device_status()
        print(f"{w.name} last chunk: {n} calls, device status {st}")
        return 0 if st == 0 else 1
    if base != w.kind:
        raise SystemExit(f"{name} is a {w.kind} workload")
    fp8 = kind.endswith("_fp8")
    page = int(kind.split("_")[1][len("paged"):]) if kind.startswith("decode_paged") else 0
    if base == "decode" and (fp8 or page):
        lens = inputs.ragged_lengths(w.seed, w.B, *w.ragged) if w.ragged else w.kv_len
        seed = w.seed * 1000 + w.n_kv if w.ragged else w.seed
        if fp8:
            q, k, v, ks, vs, lens = inputs.decode_fp8_inputs(seed, w.B, w.h, w.n_kv, w.d, lens)
            ks, vs = ks.cuda(), vs.cuda()
        else:
            q, k, v, lens = inputs.decode_inputs(seed, w.B, w.h, w.n_kv, w.d, lens)
            ks = vs = None
        if page:
            k, v, bt = inputs.page_caches(seed, k, v, lens, page)
            q, k, v, bt, lens = (x.cuda() for x in (q, k, v, bt, lens))
            call = lambda: gqa.decode_paged(q, k, v, bt, lens, k_scale=ks, v_scale=vs)  # noqa: E731
        else:
            q, k, v, lens = (x.cuda() for x in (q, k, v, lens))
            call = lambda: gqa.decode_fp8(q, k, v, ks, vs, lens)  # noqa: E731
    else:
        t = [x.cuda() for x in inputs.workload_inputs(w)]
        call = (lambda: gqa.decode(*t)) if base == "decode" else (lambda: gqa.prefill(*t, causal=w.causal))
    for _ in range(n):
        call()
    torch.cuda.synchronize()
    st = gqa.gqa_get_device_status()
    print(f"{w.name}: {n} calls, device status {st}")
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
