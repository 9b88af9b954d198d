"""bench.py host logic (CPU): the parity summary its CPU-baseline leg attaches to the line.

The leg compares a decode output with the fp64 oracle on every sequence it times.  Fed
the oracle's own result rounded to bf16 it must report every element within the bound;
one element moved by 0.05 must be caught.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

import oracle
from attention_gqa_decode_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def rounded_oracle():
    w = inputs.GQA_DECODE_70B
    q, k, v, lens = inputs.workload_inputs(w)
    return torch.from_numpy(oracle.decode(q, k, v, lens)).to(torch.bfloat16)


def test_parity_of_the_rounded_oracle_is_within_bound(bench, rounded_oracle):
    w = inputs.GQA_DECODE_70B
    cpu, parity = bench.oracle_decode_leg(target_s=0.5, gpu_out=rounded_oracle)
    assert cpu["kind"] == "oracle" and cpu["value"] > 0
    # whole sequences, each compared at most once (how many depends on the core count)
    n = parity["outputs"]
    assert n % (w.h * w.d) == 0 and w.h * w.d <= n <= w.B * w.h * w.d
    assert parity["within_bound"]
    # bf16 rounding of the output is all that separates the two: at most half a step
    assert parity["max_err_over_bound"] <= 0.5
    assert parity["mean_abs"] < 1e-4


def test_parity_catches_one_wrong_element(bench, rounded_oracle):
    bad = rounded_oracle.clone()
    bad[0, 17, 40] = float(bad[0, 17, 40]) + 0.05        # sequence 0 is in every sample
    _, parity = bench.oracle_decode_leg(target_s=0.5, gpu_out=bad)
    assert not parity["within_bound"]
    assert parity["max_err_over_bound"] > 1.0


def test_reference_leg_has_no_parity(bench):
    cpu, parity = bench.oracle_decode_leg(target_s=0.1)
    assert parity is None and np.isfinite(cpu["value"])
