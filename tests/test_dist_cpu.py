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
import sys

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


# ----------------------------------------------------------- KCP (3 ranks)
# Context parallelism across devices: rank r holds segment r of every
# sequence; the ranks exchange their fp32 segment maps and fold the earlier
# ones into their initial state.  Here the per-rank steps are the fp64 oracle
# (segment_transition, the recurrence from a given state) and a plain fold, so
# that the exchange, the rank ordering and the initial/final-state handling of
# linear_attention_recurrence_06_b200.kcp run on CPU gloo ranks.

KCP_LENS = [(21, 0, 30), (9, 40, 2)]  # per sequence: tokens on ranks 0, 1, 2 (an empty piece included)
KCP_H, KCP_D = 2, 8


class _OracleKcpBackend:
    def transition(self, q, k, v, log_alpha, beta, *, scale, cu_seqlens, max_seqlen, stream=None):
        import torch
        import oracle
        cu = cu_seqlens
        N, H, D = len(cu) - 1, k.shape[1], k.shape[2]
        trans = np.zeros((2, N, H, D, D))
        for n in range(N):
            a, b = cu[n], cu[n + 1]
            for h in range(H):
                if b > a:
                    trans[0, n, h], trans[1, n, h] = oracle.segment_transition(k[a:b, h], v[a:b, h],
                                                                               log_alpha[a:b, h], beta[a:b, h])
                else:
                    trans[0, n, h] = np.eye(D)
        return torch.from_numpy(trans), (q, k, v, log_alpha, beta, scale, cu)

    def compose(self, gathered, n_prev, initial_state, stream=None):
        g = gathered.numpy()
        s = np.zeros(g.shape[2:]) if initial_state is None else np.array(initial_state, dtype=np.float64)
        for j in range(n_prev):
            s = np.einsum("nhik,nhkc->nhic", g[j, 0], s) + g[j, 1]
        return s

    def finish(self, state_in, ctx, *, gate, norm_weight, eps, out_dtype, stream=None):
        import oracle
        q, k, v, la, b, scale, cu = ctx
        return oracle.kda_recurrent(q, k, v, la, b, state_in, cu, scale=scale, n_threads=1)


def _kcp_inputs():
    from linear_attention_recurrence_06_b200 import synth
    total = sum(sum(p) for p in KCP_LENS)
    tb = synth.tokens(11, 0, total, KCP_H, KCP_D, KCP_D, bf16=True)
    s0 = synth.states(12, len(KCP_LENS), KCP_H, KCP_D, KCP_D, std=0.5)
    # global packing: sequence after sequence; rank r's piece of each sequence
    starts, t = [], 0
    for pieces in KCP_LENS:
        starts.append(t)
        t += sum(pieces)
    return tb, s0, starts


def _kcp_local(tb, starts, rank):
    idx, cu = [], [0]
    for n, pieces in enumerate(KCP_LENS):
        a = starts[n] + sum(pieces[:rank])
        idx.extend(range(a, a + pieces[rank]))
        cu.append(cu[-1] + pieces[rank])
    idx = np.asarray(idx, dtype=np.int64)
    return idx, np.asarray(cu, dtype=np.int64)


def _kcp_worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import torch.distributed as dist

    from linear_attention_recurrence_06_b200 import kcp

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        tb, s0, starts = _kcp_inputs()
        idx, cu = _kcp_local(tb, starts, rank)
        sl = lambda x: np.ascontiguousarray(x[idx])
        o, fs = kcp.kcp_prefill(sl(tb.q), sl(tb.k), sl(tb.v), sl(tb.log_alpha), sl(tb.beta), s0, scale=0.25,
                                cu_seqlens=cu, max_seqlen=int(np.diff(cu).max()), backend=_OracleKcpBackend())
        q.put((rank, idx, o, fs))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_kcp_three_ranks_match_the_whole_sequence():
    import sys
    sys.path.insert(0, ROOT)
    import oracle

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 3, _free_port()
    procs = [ctx.Process(target=_kcp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted([q.get(timeout=180) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    tb, s0, starts = _kcp_inputs()
    cu = [0]
    for pieces in KCP_LENS:
        cu.append(cu[-1] + sum(pieces))
    o_ref, fs_ref = oracle.kda_recurrent(tb.q, tb.k, tb.v, tb.log_alpha, tb.beta, s0, np.asarray(cu), scale=0.25,
                                         n_threads=1)
    covered = np.zeros(cu[-1], dtype=bool)
    for rank, idx, o, fs in results:
        np.testing.assert_allclose(o, o_ref[idx], rtol=0, atol=1e-10)
        covered[idx] = True
    assert covered.all()
    # the last rank's state after its segment is the sequences' final state
    np.testing.assert_allclose(results[-1][3], fs_ref, rtol=0, atol=1e-10)
    # a middle rank's state is the state after the first two segments, not the final one
    assert np.abs(results[1][3] - fs_ref).max() > 1e-3


def test_bench_launches_its_own_ranks():
    """`python bench.py --gpus 2` without a launcher starts two ranks itself
    (torch.distributed.run on 127.0.0.1); in dry mode they join a gloo group and
    rank 0 reports that both formed and took part in the max-over-ranks timing."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                           "MASTER_PORT")}
    env["NCCL_DEBUG"] = "WARN"
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["ranks_reported"] == 2
    assert line["max_over_ranks"] == 2.0          # the slower (larger) of the two ranks' values
    assert line["value"] == 2 * 1.0 / 2.0e-3      # whole-job rate over the slowest rank


def test_bench_refuses_a_world_size_that_contradicts_gpus():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr
