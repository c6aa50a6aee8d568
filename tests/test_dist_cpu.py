"""Multi-rank host logic on CPU (gloo, world size 2).

The hot path partitions into independent (sequence, head) recurrences, so
ranks need no data exchange: each rank runs its own shard and only timing is
reduced (max over ranks).  These tests run two gloo ranks on the host:
  * sharding the heads of one workload over ranks reproduces the single-rank
    result exactly (the fp64 oracle stands in for the per-rank computation);
  * bench.py's max-over-ranks reduction and whole-job rate.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    import oracle
    from linear_attention_recurrence_06_b200 import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # --- head-sharded run of one workload (no exchange on the data path)
        T, H, D = 70, 4, 16
        tb = synth.tokens(7, 0, T, H, D, D, bf16=True)
        per = H // world
        heads = (rank * per, (rank + 1) * per)
        o, fs = oracle.kda_recurrent(tb.q, tb.k, tb.v, tb.log_alpha, tb.beta, heads=heads, n_threads=1)
        mine = torch.from_numpy(np.ascontiguousarray(o[:, heads[0]:heads[1]]))
        parts = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(parts, mine)  # only to check the result here
        # --- timing reduction as bench.py does it
        ms = bench.max_over_ranks(1.0 + rank, dist, "cpu")
        rate = bench.whole_job_rate(world, 8192, ms)
        q.put((rank, torch.cat(parts, dim=1).numpy(), ms, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_shard_heads_and_reduce_timing():
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from linear_attention_recurrence_06_b200 import synth

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    T, H, D = 70, 4, 16
    tb = synth.tokens(7, 0, T, H, D, D, bf16=True)
    full, _ = oracle.kda_recurrent(tb.q, tb.k, tb.v, tb.log_alpha, tb.beta, n_threads=1)
    for rank, gathered, ms, rate in results:
        np.testing.assert_array_equal(gathered, full)  # shards reproduce the whole, bit for bit
        assert ms == 2.0                                  # slowest rank's time
        assert rate == pytest.approx(2 * 8192 / 2e-3)     # all ranks' units over that time
