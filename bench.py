"""Benchmark: GQA decode KV GB/s (vs HBM peak) and causal prefill TFLOP/s (vs bf16 peak).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--split]

One JSON line on stdout (rank 0).  A step is one decode call over the whole
GQA decode workload (B=16 sequences, h=64, n_kv=8, d=128, 4096 cached tokens
each), inputs resident in device memory; three copies of the KV cache are
rotated so every step reads a cache L2 has not seen for two steps (each copy,
256 MiB, is twice the 126 MB L2).  The K decode steps are captured once in a
CUDA graph and one replay is timed between two CUDA events (the launches then
reach the GPU back to back, as in a decode serving loop); "e2e" times the
public API call with its host copies instead.

The same run times, each under its own key:
  prefill                 the causal prefill workload (B=4, S=4096, h=32, n_kv=8, d=128)
  prefill_paged_chunk     its last 512-token chunk over a paged cache, with the append
  decode_mqa              the MQA decode workload (B=64, h=32, n_kv=1, d=128, L=8192)
  decode_ragged_nkv{64,8,1}  the ragged decode sweep (B=32, h=64, d=128, lengths
                          uniform on [512, 8192]), with the KV bytes one decoded
                          token of a sequence reads (2 * 2 * n_kv * d * L_b)
  decode_fp8, decode_paged, decode_paged_fp8, decode_fp8_mqa
                          the GQA (and MQA) decode workloads over E4M3 and paged caches
  mla_decode              absorbed MLA decode (B=16, h=32, d_c=512, L=4096)
  mla_decode_long         absorbed MLA decode (B=4, h=32, d_c=512, L=65536; the tcgen05 kernel)
Under torchrun every rank runs the same per-GPU workload (the (sequence, KV
head) units are independent: weak scaling, no collective on the data path);
with --split the decode workload's batch is divided among the ranks instead
(strong scaling).  The time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_gqa_decode_b200 import multirank  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
N_KV_COPIES = 3


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        mp = json.load(open(path))
        return {"hbm": float(mp["hbm_gbs"]), "bf16": float(mp["bf16_tflops"]),
                "bf16_sustained": float(mp.get("bf16_tflops_sustained", mp["bf16_tflops"])), "src": "measured"}
    except Exception:
        return {"hbm": FALLBACK_HBM_GBS, "bf16": FALLBACK_BF16_TFLOPS, "bf16_sustained": 1400.0, "src": "fallback"}


# the committed ncu traffic record of the decode launch each named leg times (the split
# path's merge kernel is not included: 5.9 MB of L2-resident partials at MQA B64)
NAMED_TRAFFIC = {"decode_mqa": "gqa_decode_bal_kernel[mqa]",
                 "decode_ragged_nkv64": "gqa_decode_kernel[ragged n_kv64]",
                 "decode_ragged_nkv8": "gqa_decode_kernel[ragged n_kv8]",
                 "decode_ragged_nkv1": "gqa_decode_bal_kernel[ragged n_kv1]"}


def kernel_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if its source hash is current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel]
    except Exception:
        return None
    src = os.path.join(ROOT, rec["source"])
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    return rec["bytes_per_launch"] if h == rec["source_sha256"] else None


class ClockSampler:
    """SM clock and throttle reasons, sampled through NVML while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, device, period_s: float = 0.01):
        self.device, self.period = device, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            import torch
            pr = torch.cuda.get_device_properties(self.device)
            bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._nv = None
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------
# CPU legs (the oracle, as it stands, on the host cores)

def oracle_decode_leg(target_s: float = 10.0, gpu_out=None):
    """Time the fp64 oracle on whole sequences of the decode workload until ~target_s.

    With `gpu_out` (the decode leg's bf16 result for the same seeded inputs) every
    output of the sequences the oracle computed is also compared with it; the
    comparison is returned as a second dict (None without `gpu_out`)."""
    import numpy as np
    import oracle
    import torch
    from attention_gqa_decode_b200 import inputs, metrics
    w = inputs.GQA_DECODE_70B
    from tests import _tol
    q, k, v, lens = inputs.workload_inputs(w)
    vmax = _tol.value_absmax(v)
    per_seq = w.kv_len
    cores = os.cpu_count() or 1
    done_bytes, t_total, seqs = 0, 0.0, 0
    b = 0
    errs, ulps, over, seen = [], [], 0, set()
    while t_total < target_s and seqs < 4 * w.B:
        nb = min(cores, w.B)                      # one batch of sequences per call, all cores
        b0 = (b * nb) % w.B
        idx = [(b0 + i) % w.B for i in range(nb)]
        qs = q[idx].contiguous()
        ks = torch.cat([k[j * per_seq:(j + 1) * per_seq] for j in idx]).contiguous()
        vs = torch.cat([v[j * per_seq:(j + 1) * per_seq] for j in idx]).contiguous()
        ls = lens[idx].contiguous()
        t0 = time.perf_counter()
        ref = oracle.decode(qs, ks, vs, ls, n_threads=cores)
        t_total += time.perf_counter() - t0
        done_bytes += metrics.decode_kv_bytes(ls.tolist(), w.n_kv, w.d)
        seqs += nb
        b += 1
        fresh = [i for i, j in enumerate(idx) if j not in seen]   # each sequence compared once
        if gpu_out is not None and fresh:
            seen.update(idx[i] for i in fresh)
            got = gpu_out[[idx[i] for i in fresh]].double().numpy()
            ref = ref[fresh]
            err = np.abs(got - ref)
            lim = _tol.bound(ref, vmax, w.kv_len)
            errs.append(err.ravel())
            ulps.append((err / lim).ravel())
            over += int((err > lim).sum())
    cpu = {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
           "sample": f"{seqs} whole sequences of the decode workload ({w.kv_len} tokens, h={w.h}, n_kv={w.n_kv}), "
                     f"{t_total:.1f} s of fp64 oracle time"}
    if not errs:
        return cpu, None
    e, u = np.concatenate(errs), np.concatenate(ulps)
    parity = {"outputs": int(e.size), "max_abs": float(e.max()), "mean_abs": float(e.mean()),
              "max_err_over_bound": float(u.max()),
              "above_1e-2": int((e > _tol.MAX_ABS).sum()),
              "within_bound": bool(over == 0 and e.mean() <= _tol.MEAN_ABS),
              "bound": "|gpu - oracle| <= 1e-2 where |oracle| < 4, else half a bf16 step + weight rounding "
                       "+ fp32 sums (derived in tests/_tol.py); mean <= 1e-3",
              "what": "the timed decode leg's output against the fp64 oracle on the sequences of the CPU sample"}
    return cpu, parity


# ----------------------------------------------------------------------------
# GPU legs

def time_steps(fn, steps, warmup, stream):
    """CUDA-event time (ms) of `steps` calls fn(step), after `warmup` untimed calls.

    The steps are captured once into a CUDA graph (fn launches through the C ABI
    on torch's current stream, which is the capture stream), the graph is
    replayed once untimed, then once between two events, synchronised on both
    sides: the launches reach the GPU back to back, without the per-call host
    path between them (the serving loop of a decoder runs the same way)."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    g.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    del g
    return t0.elapsed_time(t1)


def time_launches(fn, steps, warmup, stream, flush=None):
    """CUDA-event time of each launch of fn(step) on `stream`; returns per-step ms list and total ms."""
    import torch
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    tot0, tot1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tot0.record(stream)
    for i in range(steps):
        if flush is not None:
            flush(i)
        ev[i][0].record(stream)
        fn(i)
        ev[i][1].record(stream)
    tot1.record(stream)
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in ev]
    return per, tot0.elapsed_time(tot1)


def decode_leg(args, device, world, clocks):
    import torch
    import attention_gqa_decode_b200 as gqa
    from attention_gqa_decode_b200 import inputs, metrics
    w = inputs.GQA_DECODE_70B
    q, k, v, lens = inputs.workload_inputs(w)
    if args.split and world > 1:
        # strong scaling: this rank's shard of the one global batch (sequences [lo, hi))
        rank = int(os.environ.get("RANK", 0))
        lo, hi, r0, r1 = multirank.packed_shard(lens.tolist(), rank, world)
        q, k, v, lens = (q[lo:hi].contiguous(), k[r0:r1].contiguous(), v[r0:r1].contiguous(),
                         lens[lo:hi].contiguous())
    kv_bytes = metrics.decode_kv_bytes(lens.tolist(), w.n_kv, w.d)
    qd, ld = q.to(device), lens.to(device)
    ks = [k.to(device) for _ in range(N_KV_COPIES)]
    vs = [v.to(device) for _ in range(N_KV_COPIES)]
    out = torch.empty_like(qd)
    stream = torch.cuda.current_stream(device)

    def step(i):
        c = i % N_KV_COPIES
        gqa.decode(qd, ks[c], vs[c], ld, out=out)

    barrier(world)
    torch.cuda.synchronize()
    with clocks:
        total = time_steps(step, args.steps, args.warmup, stream)
    barrier(world)
    total_max = multirank.max_over_ranks(total, device)
    # the decode kernel is the only kernel in the timed region: its average launch
    # duration there is total / steps.  (Events around each launch, timed apart,
    # also show the idle gap they force between launches.)
    kern_ms = total_max / args.steps
    per, _ = time_launches(step, min(args.steps, 100), 3, stream)
    res_isolated = statistics.mean(per)
    st = gqa.gqa_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the decode leg")
    res = {"kv_bytes": kv_bytes, "total_ms": total_max, "kernel_ms": kern_ms, "isolated_ms": res_isolated,
           "out": out.cpu()}   # the timed steps' result (every cache copy holds the same values)

    # end to end through the public API: pinned host inputs -> device -> decode -> host result
    qh, kh, vh, lh = (t.pin_memory() for t in (q, k, v, lens))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    qe, ke, ve, le = (torch.empty_like(t, device=device) for t in (q, k, v, lens))
    e2e_steps = max(3, min(10, args.steps))

    def e2e(i):
        qe.copy_(qh, non_blocking=True)
        ke.copy_(kh, non_blocking=True)
        ve.copy_(vh, non_blocking=True)
        le.copy_(lh, non_blocking=True)
        o = gqa.decode(qe, ke, ve, le)
        oh.copy_(o, non_blocking=True)

    barrier(world)
    per_e, total_e = time_launches(e2e, e2e_steps, 2, stream)
    barrier(world)
    total_e = multirank.max_over_ranks(total_e, device)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v, lens))
    d2h = oh.numel() * oh.element_size()
    res["e2e"] = {"value": multirank.job_throughput(kv_bytes * e2e_steps, total_e, device) / 1e9, "unit": "GB/s",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    return res


def cache_variant_leg(kind, args, device, world, page_size=64):
    """The GQA decode workload over another cache: "fp8" (packed E4M3, one scale
    per KV head), "paged" (bf16, pages of `page_size` tokens in a seeded random
    order) or "paged_fp8".  Copies rotated so each step reads a cache L2 has not
    seen for two steps; CUDA-event time per launch."""
    import torch
    import attention_gqa_decode_b200 as gqa
    from attention_gqa_decode_b200 import inputs, metrics
    w = inputs.GQA_DECODE_70B
    fp8 = kind.endswith("fp8")
    if fp8:
        q, k, v, ksc, vsc, lens = inputs.decode_fp8_inputs(w.seed, w.B, w.h, w.n_kv, w.d, w.kv_len)
        ksc, vsc = ksc.to(device), vsc.to(device)
    else:
        q, k, v, lens = inputs.workload_inputs(w)
        ksc = vsc = None
    bt = None
    if kind.startswith("paged"):
        k, v, bt = inputs.page_caches(w.seed, k, v, lens, page_size)
        bt = bt.to(device)
    kv_bytes = metrics.decode_kv_bytes(lens.tolist(), w.n_kv, w.d) // (2 if fp8 else 1)
    copies = max(3, -(-3 * 128 * 1024 * 1024 // kv_bytes))   # every copy set is >= 3 x 128 MiB
    qd, ld = q.to(device), lens.to(device)
    ks = [k.to(device) for _ in range(copies)]
    vs = [v.to(device) for _ in range(copies)]
    out = torch.empty_like(qd)
    stream = torch.cuda.current_stream(device)

    def step(i):
        c = i % copies
        if bt is not None:
            gqa.decode_paged(qd, ks[c], vs[c], bt, ld, k_scale=ksc, v_scale=vsc, out=out)
        else:
            gqa.decode_fp8(qd, ks[c], vs[c], ksc, vsc, ld, out=out)

    steps = max(3, min(args.steps, 300))
    barrier(world)
    total = time_steps(step, steps, max(3, args.warmup), stream)
    barrier(world)
    kern_ms = multirank.max_over_ranks(total, device) / steps
    if gqa.gqa_get_device_status() != 0:
        raise RuntimeError(f"device status after the {kind} decode leg")
    return {"kv_bytes": kv_bytes, "kernel_ms": kern_ms, "steps": steps, "copies": copies}


def named_decode_leg(args, device, world, w, fp8=False):
    """A named decode workload (packed bf16 cache, or E4M3 with one scale per KV
    head), K steps graph-timed like the headline leg; cache copies rotated so
    every copy set is >= 3 x 128 MiB (each step reads a cache L2 has not seen
    for two steps).  Reports KV GB/s and the KV bytes one decoded token of a
    sequence reads, 2 * b * n_kv * d_h * L_b (the cache formula with one layer
    and B = 1)."""
    import torch
    import attention_gqa_decode_b200 as gqa
    from attention_gqa_decode_b200 import inputs, metrics
    lens = inputs.ragged_lengths(w.seed, w.B, *w.ragged) if w.ragged else w.kv_len
    seed = w.seed * 1000 + w.n_kv if w.ragged else w.seed
    if fp8:
        q, k, v, ksc, vsc, lens = inputs.decode_fp8_inputs(seed, w.B, w.h, w.n_kv, w.d, lens)
        ksc, vsc = ksc.to(device), vsc.to(device)
    else:
        q, k, v, lens = inputs.decode_inputs(seed, w.B, w.h, w.n_kv, w.d, lens)
    eb = 1 if fp8 else 2
    per_token = [metrics.decode_kv_bytes([int(x)], w.n_kv, w.d, eb) for x in lens.tolist()]
    kv_bytes = sum(per_token)
    copies = max(3, -(-3 * 128 * 1024 * 1024 // kv_bytes))
    qd, ld = q.to(device), lens.to(device)
    ks = [k.to(device) for _ in range(copies)]
    vs = [v.to(device) for _ in range(copies)]
    del k, v
    out = torch.empty_like(qd)
    stream = torch.cuda.current_stream(device)

    def step(i):
        c = i % copies
        if fp8:
            gqa.decode_fp8(qd, ks[c], vs[c], ksc, vsc, ld, out=out)
        else:
            gqa.decode(qd, ks[c], vs[c], ld, out=out)

    steps = max(3, min(args.steps, 300))
    barrier(world)
    total = time_steps(step, steps, max(3, args.warmup), stream)
    barrier(world)
    kern_ms = multirank.max_over_ranks(total, device) / steps
    if gqa.gqa_get_device_status() != 0:
        raise RuntimeError(f"device status after the {w.name} leg")
    del ks, vs
    torch.cuda.empty_cache()
    return {"kv_bytes": kv_bytes, "kernel_ms": kern_ms, "steps": steps, "copies": copies, "B": w.B,
            "bytes_per_token": {"mean": kv_bytes / w.B, "min": min(per_token), "max": max(per_token)}}


def chunk_prefill_leg(args, device, world):
    """The last 512-token chunk of B=4 sequences of 4096 tokens (h=32, n_kv=8, d=128):
    3584 past tokens in 64-token pages (seeded random order), append + causal
    attention in one launch.  Each step restores nothing: the append rewrites the
    same slots with the same values."""
    import torch
    import attention_gqa_decode_b200 as gqa
    from attention_gqa_decode_b200 import inputs, metrics
    B, S_q, P, h, n_kv, d, ps = 4, 512, 3584, 32, 8, 128, 64
    q, kn, vn, kp, vp, bt, past = inputs.chunk_prefill_inputs(4, B, S_q, [P] * B, h, n_kv, d, ps)
    flops = metrics.chunk_prefill_flops([P] * B, S_q, h, d)
    qd, knd, vnd, kpd, vpd, btd, pd = (t.to(device) for t in (q, kn, vn, kp, vp, bt, past))
    out = torch.empty_like(qd)
    stream = torch.cuda.current_stream(device)
    scratch = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)   # > L2: flushed between steps

    def flush(i):
        scratch.fill_(i & 0xFF)

    steps = max(3, min(args.steps, 30))
    barrier(world)
    per, _ = time_launches(lambda i: gqa.prefill_paged(qd, knd, vnd, kpd, vpd, btd, pd, out=out), steps,
                           max(3, args.warmup), stream, flush=flush)
    barrier(world)
    kern_ms = multirank.max_over_ranks(statistics.mean(per), device)
    if gqa.gqa_get_device_status() != 0:
        raise RuntimeError("device status after the chunked prefill leg")
    return {"flops": flops, "kernel_ms": kern_ms, "steps": steps,
            "workload": f"chunked prefill B{B} S_q{S_q} past{P} h{h} n_kv{n_kv} d{d}, {ps}-token pages"}


def mla_leg(args, device, world, w=None):
    """Absorbed MLA decode, B16 h32 d_c512 L4096 (64 MiB latent cache per step) unless
    another MLA workload is given; copies rotated so each step reads a cache L2 has not
    seen for several steps."""
    import torch
    import attention_gqa_decode_b200 as gqa
    from attention_gqa_decode_b200 import inputs
    w = w or inputs.MLA_DECODE
    q, c, lens = inputs.mla_decode_inputs(w.seed, w.B, w.h, w.d, w.kv_len)
    nbytes = c.numel() * c.element_size()
    copies = max(3, -(-3 * 128 * 1024 * 1024 // nbytes))
    qd, ld = q.to(device), lens.to(device)
    cs = [c.to(device) for _ in range(copies)]
    out = torch.empty_like(qd)
    stream = torch.cuda.current_stream(device)
    steps = max(3, min(args.steps, 300))
    barrier(world)
    total = time_steps(lambda i: gqa.mla_decode(qd, cs[i % copies], ld, out=out), steps, max(3, args.warmup), stream)
    barrier(world)
    kern_ms = multirank.max_over_ranks(total, device) / steps
    if gqa.gqa_get_device_status() != 0:
        raise RuntimeError("device status after the MLA decode leg")
    return {"kv_bytes": nbytes, "kernel_ms": kern_ms, "steps": steps, "copies": copies, "workload": w.name,
            "B": w.B, "path": gqa.gqa_mla_decode_path(w.B, w.h, w.d, int(lens.clamp(min=0).sum()), 1)}


def prefill_leg(args, device, world):
    import torch
    import attention_gqa_decode_b200 as gqa
    from attention_gqa_decode_b200 import inputs, metrics
    w = inputs.GQA_CAUSAL_PREFILL
    q, k, v = inputs.workload_inputs(w)
    flops = metrics.prefill_flops(w.B, w.S_q, w.S_kv, w.h, w.d, True)
    qd, kd, vd = q.to(device), k.to(device), v.to(device)
    out = torch.empty_like(qd)
    stream = torch.cuda.current_stream(device)
    scratch = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)   # > L2: flushed between steps

    def flush(i):
        scratch.fill_(i & 0xFF)

    steps = max(3, min(args.steps, 30))
    barrier(world)
    per, _ = time_launches(lambda i: gqa.prefill(qd, kd, vd, causal=True, out=out), steps, max(3, args.warmup),
                           stream, flush=flush)
    barrier(world)
    kern_ms = multirank.max_over_ranks(statistics.mean(per), device)
    if gqa.gqa_get_device_status() != 0:
        raise RuntimeError("device status after the prefill leg")
    return {"flops": flops, "kernel_ms": kern_ms, "steps": steps,
            "io_bytes": metrics.prefill_io_bytes(w.B, w.S_q, w.S_kv, w.h, w.n_kv, w.d)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true", help="skip the E4M3 / paged cache legs")
    ap.add_argument("--no-sweep", action="store_true", help="skip the MQA and ragged-sweep decode legs")
    ap.add_argument("--split", action="store_true",
                    help="under torchrun, split the decode workload's batch across the ranks (strong scaling) "
                         "instead of running the per-GPU workload on every rank (weak scaling)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local = dist_env()
    from attention_gqa_decode_b200 import inputs
    w = inputs.GQA_DECODE_70B
    metric = "GQA decode KV GB/s"
    split = args.split and world > 1
    config = {"workload": w.name, "B": w.B, "h": w.h, "n_kv": w.n_kv, "d_h": w.d, "kv_len": w.kv_len,
              "global_batch": w.B if split else w.B * world, "parallelism": f"dp{world}" if world > 1 else "single",
              "l2": f"{N_KV_COPIES} KV copies of 256 MiB rotated (each step reads a cache unseen for 2 steps)",
              "timing": "K steps captured in a CUDA graph, one replay between two CUDA events on the launching stream"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        cpu, _ = oracle_decode_leg(target_s=min(60.0, 5.0 + 0.2 * args.steps))
        line = {"impl": "reference", "metric": metric, "value": cpu["value"], "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) bf16 inputs)",
                "config": config, "cpu_baseline": cpu,
                "e2e": {"value": cpu["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    pk = peaks()
    clocks = ClockSampler(device)
    dec = decode_leg(args, device, world, clocks)
    pre = None if args.no_prefill else prefill_leg(args, device, world)
    chunk = None if (args.no_prefill or args.no_variants) else chunk_prefill_leg(args, device, world)
    mla = None if args.no_variants else mla_leg(args, device, world)
    mla_long = None if args.no_variants else mla_leg(args, device, world, inputs.MLA_DECODE_LONG)
    variants = {} if args.no_variants else {
        "decode_fp8": cache_variant_leg("fp8", args, device, world),
        "decode_paged": cache_variant_leg("paged", args, device, world),
        "decode_paged_fp8": cache_variant_leg("paged_fp8", args, device, world),
    }
    named = {}
    if not args.no_sweep:
        named["decode_mqa"] = (inputs.MQA_DECODE_LONG, False, named_decode_leg(args, device, world,
                                                                               inputs.MQA_DECODE_LONG))
        for wr in inputs.RAGGED_SWEEP:
            named[f"decode_ragged_nkv{wr.n_kv}"] = (wr, False, named_decode_leg(args, device, world, wr))
        if not args.no_variants:
            named["decode_fp8_mqa"] = (inputs.MQA_DECODE_LONG, True, named_decode_leg(args, device, world,
                                                                                      inputs.MQA_DECODE_LONG, True))

    value = multirank.job_throughput(dec["kv_bytes"] * args.steps, dec["total_ms"], device) / 1e9
    achieved = dec["kv_bytes"] / (dec["kernel_ms"] / 1e3) / 1e9
    line = {
        "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dec["total_ms"] / args.steps, "higher_is_better": True,
        "scaling": "strong" if split else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v)", "config": config,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                     "frac": achieved / pk["hbm"], "traffic": kernel_traffic("gqa_decode_kernel"),
                     "algorithmic_bytes_per_launch": dec["kv_bytes"], "peak_source": pk["src"],
                     "launch_ms": dec["kernel_ms"], "launch_ms_isolated": dec["isolated_ms"]},
        "e2e": dec["e2e"],
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    if pre is not None:
        tf = pre["flops"] / (pre["kernel_ms"] / 1e3) / 1e12
        line["prefill"] = {
            "metric": "GQA causal prefill TFLOP/s", "workload": inputs.GQA_CAUSAL_PREFILL.name,
            "value": world * tf, "unit": "TFLOP/s", "ms_per_call": pre["kernel_ms"], "steps": pre["steps"],
            "l2": "256 MiB buffer written between calls",
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16"], "unit": "TFLOP/s",
                         "frac": tf / pk["bf16"], "frac_of_sustained": tf / pk["bf16_sustained"],
                         "traffic": kernel_traffic("gqa_prefill_kernel"),
                         "algorithmic_flops_per_launch": pre["flops"], "peak_source": pk["src"]}}
    if chunk is not None:
        tf = chunk["flops"] / (chunk["kernel_ms"] / 1e3) / 1e12
        line["prefill_paged_chunk"] = {
            "metric": "GQA causal prefill TFLOP/s", "workload": chunk["workload"], "value": world * tf,
            "unit": "TFLOP/s", "ms_per_call": chunk["kernel_ms"], "steps": chunk["steps"],
            "l2": "256 MiB buffer written between calls",
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16"], "unit": "TFLOP/s",
                         "frac": tf / pk["bf16"], "traffic": kernel_traffic("gqa_prefill_kernel[paged]"),
                         "algorithmic_flops_per_launch": chunk["flops"], "peak_source": pk["src"]}}
    for key, r, tk in (("mla_decode", mla, "gqa_mla_decode_kernel"),
                       ("mla_decode_long", mla_long, "mla_decode_tc_kernel[long]")):
        if r is None:
            continue
        gbs = r["kv_bytes"] / (r["kernel_ms"] / 1e3) / 1e9
        line[key] = {
            "metric": "MLA decode latent-cache GB/s", "workload": r["workload"], "value": world * gbs,
            "unit": "GB/s", "ms_per_call": r["kernel_ms"], "steps": r["steps"],
            "kernel": {0: "warp-level MMA", 1: "tcgen05, splits merged in a cluster",
                       2: "tcgen05, splits merged through a workspace"}.get(r["path"], "unknown"),
            "tokens_per_s": world * r["B"] / (r["kernel_ms"] / 1e3), "l2": f"{r['copies']} cache copies rotated",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s", "frac": gbs / pk["hbm"],
                         "traffic": kernel_traffic(tk),
                         "algorithmic_bytes_per_launch": r["kv_bytes"], "peak_source": pk["src"]}}
    desc = {"decode_fp8": ("E4M3 cache, one fp32 scale per KV head", "gqa_decode_kernel[e4m3]"),
            "decode_paged": ("bf16 cache in 64-token pages, seeded random page order", "gqa_decode_kernel[paged]"),
            "decode_paged_fp8": ("E4M3 cache in 64-token pages", "gqa_decode_kernel[paged,e4m3]")}
    for name, r in variants.items():
        gbs = r["kv_bytes"] / (r["kernel_ms"] / 1e3) / 1e9
        line[name] = {
            "metric": "GQA decode KV GB/s", "workload": f"{w.name}, {desc[name][0]}",
            "value": world * gbs, "unit": "GB/s", "ms_per_call": r["kernel_ms"], "steps": r["steps"],
            "tokens_per_s": world * w.B / (r["kernel_ms"] / 1e3),
            "l2": f"{r['copies']} cache copies rotated",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": gbs / pk["hbm"], "traffic": kernel_traffic(desc[name][1]),
                         "algorithmic_bytes_per_launch": r["kv_bytes"], "peak_source": pk["src"]}}
    for name, (wn, fp8, r) in named.items():
        gbs = r["kv_bytes"] / (r["kernel_ms"] / 1e3) / 1e9
        line[name] = {
            "metric": "GQA decode KV GB/s", "workload": wn.name + (", E4M3 cache, one fp32 scale per KV head"
                                                                   if fp8 else ""),
            "value": world * gbs, "unit": "GB/s", "ms_per_call": r["kernel_ms"], "steps": r["steps"],
            "tokens_per_s": world * r["B"] / (r["kernel_ms"] / 1e3),
            "kv_bytes_per_decoded_token": r["bytes_per_token"],
            "l2": f"{r['copies']} cache copies rotated",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": gbs / pk["hbm"], "traffic": kernel_traffic(NAMED_TRAFFIC.get(name, "")),
                         "algorithmic_bytes_per_launch": r["kv_bytes"], "peak_source": pk["src"]}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], parity = oracle_decode_leg(target_s=10.0, gpu_out=dec["out"])
        if parity is not None:
            line["parity"] = parity
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
