"""The N > 1 host path on CPU: two gloo ranks, 127.0.0.1 rendezvous.

The decode path shards by batch with no exchange on the data path: each rank
attends its own sequences, and the results are disjoint slices.  The split is
checked end to end on the ragged decode sweep's batch: each rank runs the fp64
oracle on its shard (multirank.packed_shard), the shards are gathered over
gloo, and the result equals the unsharded oracle bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from attention_gqa_decode_b200 import inputs, multirank


def test_shard_range_partitions():
    for n in (0, 1, 5, 16, 17, 1000):
        for world in (1, 2, 3, 8):
            spans = [multirank.shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        multirank.shard_range(4, 2, 2)


def test_single_process_reductions_are_identity():
    assert multirank.max_over_ranks(3.5) == 3.5
    assert multirank.job_throughput(10.0, 2.0) == 10.0 / 0.002


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lo, hi = multirank.shard_range(33, rank, world)
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slowest
        out = (multirank.max_over_ranks(ms), multirank.sum_over_ranks(hi - lo),
               multirank.job_throughput(hi - lo, ms))
        dist.barrier()
        q.put((rank, lo, hi, out))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [(lo, hi) for _, lo, hi, _ in res] == [(0, 17), (17, 33)]
    for _, _, _, (mx, tot, thr) in res:
        assert mx == 15.0 and tot == 33.0
        assert abs(thr - 33.0 / 0.015) < 1e-6


def test_packed_shard_covers_the_rows():
    lens = [5, 0, -3, 7, 1, 9, 2]
    for world in (1, 2, 3, 7):
        spans = [multirank.packed_shard(lens, r, world) for r in range(world)]
        assert spans[0][:1] == (0,) and spans[-1][1] == len(lens)
        assert spans[0][2] == 0 and spans[-1][3] == sum(max(x, 0) for x in lens)
        for (lo, hi, r0, r1), nxt in zip(spans, spans[1:] + [None]):
            assert r1 - r0 == sum(max(x, 0) for x in lens[lo:hi])
            if nxt is not None:
                assert (hi, r1) == (nxt[0], nxt[2])


# the ragged sweep's batch (32 sequences, lengths uniform on [512, 8192]) at its
# single-KV-head point, with fewer query heads so the oracle stays quick
SPLIT_H, SPLIT_NKV = 8, 1


def _split_inputs():
    w = inputs.RAGGED_SWEEP[-1]
    lens = inputs.ragged_lengths(w.seed, w.B, *w.ragged)
    return inputs.decode_inputs(w.seed * 1000 + SPLIT_NKV, w.B, SPLIT_H, SPLIT_NKV, w.d, lens)


def _split_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        qq, k, v, lens = _split_inputs()
        lo, hi, r0, r1 = multirank.packed_shard(lens.tolist(), rank, world)
        part = torch.from_numpy(oracle.decode(qq[lo:hi].contiguous(), k[r0:r1].contiguous(), v[r0:r1].contiguous(),
                                              lens[lo:hi].contiguous(), n_threads=2))
        sizes = [multirank.shard_range(len(lens), r, world) for r in range(world)]
        bufs = [torch.empty((b - a,) + tuple(part.shape[1:]), dtype=torch.float64) for a, b in sizes]
        if rank == 0:
            dist.gather(part, bufs, dst=0)
            q.put(torch.cat(bufs).numpy())
        else:
            dist.gather(part, None, dst=0)
    finally:
        dist.destroy_process_group()


def test_batch_split_over_two_gloo_ranks_equals_unsharded():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered = q.get(timeout=300)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    qq, k, v, lens = _split_inputs()
    whole = oracle.decode(qq, k, v, lens)
    assert gathered.shape == whole.shape
    assert np.array_equal(gathered, whole)
