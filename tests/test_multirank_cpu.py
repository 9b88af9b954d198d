"""The N > 1 host path on CPU: two gloo ranks, 127.0.0.1 rendezvous."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from attention_gqa_decode_b200 import multirank


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
