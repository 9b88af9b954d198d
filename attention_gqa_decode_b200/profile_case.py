"""Run a named workload a few times on cuda:0, for profilers (ncu -k ... -s ... -c ...).

    python -m attention_gqa_decode_b200.profile_case decode GQA_DECODE_70B 3
    python -m attention_gqa_decode_b200.profile_case prefill GQA_CAUSAL_PREFILL 2
    python -m attention_gqa_decode_b200.profile_case decode RAGGED_SWEEP:2 3

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
    if kind != w.kind:
        raise SystemExit(f"{name} is a {w.kind} workload")
    t = [x.cuda() for x in inputs.workload_inputs(w)]
    for _ in range(n):
        if kind == "decode":
            gqa.decode(*t)
        else:
            gqa.prefill(*t, causal=w.causal)
    torch.cuda.synchronize()
    st = gqa.gqa_get_device_status()
    print(f"{w.name}: {n} calls, device status {st}")
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
