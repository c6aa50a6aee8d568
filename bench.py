#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200.

Headline (one "step"): one chunkwise prefill call of the KDA recurrence over
B=1, T=8192, H=32, dk=dv=128, bf16 inputs, fp32 state, 64-token chunks, with
the per-head RMSNorm and sigmoid output gate (kda_chunk_fwd with gate).
Reported as whole-job tokens/s (weak scaling: every rank runs its own batch),
plus TFLOP/s against the dense BF16 tensor peak and the call's HBM roofline.
A decode sub-measurement runs 1000 consecutive recurrent steps over 256
sequences x 32 heads (fp32 state, 512 MiB) and reports steps/s and state GB/s
against HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1: one rank per GPU over NCCL.  Launched under torch.distributed.run the
script uses its RANK / WORLD_SIZE; launched plainly with --gpus N it starts the
N ranks itself through torch.distributed.run.  Rank 0 prints ONE JSON line.  `--impl reference` times the fp64 CPU oracle (the only
reference implementation that exists for this method) on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (TFLOP/s, % peak); decode steps/s (state GB/s, % HBM)"
D = 128
PREFILL = dict(B=1, T=8192, H=32)
DECODE = dict(Bd=256, H=32, steps=1000, pool=8)
# algorithmic work per token-head (chunk 64, dk = dv = 128):
#   bytes: q, k, v, log_alpha, gate in + y out (6 x 256 B bf16) + beta (2 B)
#   flops: C^2 (3 dk + 2 dv) triangular intra-chunk products + 6 C dk dv state products, per chunk of C
PREFILL_BYTES_PER_TH = 6 * 256 + 2
PREFILL_FLOP_PER_TH = 139264
DECODE_STATE_BYTES_PER_HEAD = 2 * D * D * 4
DECODE_TOKEN_BYTES_PER_HEAD = 4 * 256 + 2 + 256   # q, k, v, log_alpha in; beta; o out
WORKLOAD = ("KDA chunkwise prefill, B=1 T=8192 H=32 dk=dv=128, bf16 inputs, fp32 state, chunk 64, "
            "fused per-head RMSNorm + sigmoid gate, zero initial state")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """Largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(n_ranks: int, units_per_rank: float, ms_max: float) -> float:
    """Weak scaling: every rank processes its own units; the job's rate is all
    units over the slowest rank's time."""
    return n_ranks * units_per_rank / (ms_max * 1e-3)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is under load."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for ln in out.strip().splitlines():
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append(dict(sm=float(parts[0]), smax=float(parts[1]), reasons=parts[3:8]))
            except ValueError:
                continue
        if not rows:
            return None
        smax = max(r["smax"] for r in rows)
        loaded = [r for r in rows if r["sm"] > 0.3 * smax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for r in loaded:
            for nm, val in zip(names, r["reasons"][1:]):
                if val.lower().startswith("active"):
                    seen.add(nm)
        return dict(sm_mhz=statistics.median(r["sm"] for r in loaded), sm_max_mhz=smax, reasons=sorted(seen),
                    samples=len(loaded))


# -------------------------------------------------------------------- inputs

def prefill_inputs(seed: int):
    from linear_attention_recurrence_06_b200 import synth
    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    tb = synth.tokens(seed, 0, B * T, H, D, D, bf16=True, gate=True)
    return tb


def to_bf16_host(a, torch, pin=True):
    t = torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)
    return t.pin_memory() if pin else t


# ----------------------------------------------------------------- our arm

def run_ours(args, peaks):
    import torch
    import linear_attention_recurrence_06_b200 as kda

    ws_n, rank, local = dist_env()
    dist = None
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        # NCCL prints its communicator set-up, so the number of ranks that formed is on record
        os.environ.setdefault("NCCL_DEBUG", "INFO")
        os.environ.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    def mor(x: float) -> float:
        return max_over_ranks(x, dist, dev)

    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    tb = prefill_inputs(seed=rank)
    hq = {n: to_bf16_host(getattr(tb, n).reshape(B, T, H, -1) if n != "beta" else tb.beta.reshape(B, T, H), torch)
          for n in ("q", "k", "v", "log_alpha", "beta", "g")}
    dq = {n: t.to(dev) for n, t in hq.items()}
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    _, ws_full = kda.workspace_size(B * T, H, B, T)
    ws = torch.empty(ws_full, dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_fwd(dq["q"], dq["k"], dq["v"], dq["log_alpha"], dq["beta"], None, gate=dq["g"], out=out,
                      final_state=fs, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kda.query_status(ws) != 0:
        raise RuntimeError("device status word set during warm-up")

    # per-kernel device time (events around each launch, same stream), separate pass
    kda.profile_enable(True)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    prof = kda.profile_read()
    kda.profile_enable(False)
    launches_per_step = sum(v[0] for v in prof.values()) / args.steps

    # timed region: clocks sampled over a pre-roll plus the K timed steps
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    t_end = time.time() + 1.0
    while time.time() < t_end:
        for _ in range(20):
            step()
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_step = mor(e0.elapsed_time(e1) / args.steps)

    # decode sub-measurement: 1000 consecutive steps, state in place
    dec = run_decode(args, torch, kda, dev, stream, rank, mor, barrier)
    clocks = sampler.stop() if sampler else None

    # end to end through the public API: pinned host inputs -> device -> call -> host output
    e2e = run_e2e(args, torch, kda, hq, out, fs, ws, stream, mor, barrier)

    # segment-parallel prefill on a low-parallelism shape (one sequence, one head)
    seg = run_segmented(args, torch, kda, dev, stream, mor, barrier)

    # per-device steps of context parallelism across devices (ranks emulated on this GPU)
    kcp = run_kcp(args, torch, kda, dev, stream, mor, barrier)
    if ws_n > 1:  # and across the ranks of this job: one sequence split over all of them
        kcp["across_ranks"] = run_kcp_ranks(args, torch, kda, dev, stream, rank, ws_n, mor, barrier)

    # backward of the prefill on the same shape
    bwd = run_backward(args, torch, kda, dev, stream, mor, barrier)

    # the packed varlen and the long-context workloads
    torch.cuda.empty_cache()
    varlen = run_varlen(args, torch, kda, dev, stream, mor, barrier)
    torch.cuda.empty_cache()
    long_ctx = run_long(args, torch, kda, dev, stream, mor, barrier)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    value = whole_job_rate(ws_n, B * T, ms_step)
    th = B * T * H
    bytes_call = PREFILL_BYTES_PER_TH * th
    achieved_gbs = bytes_call / (ms_step * 1e-3) / 1e9
    tflops = PREFILL_FLOP_PER_TH * th / (ms_step * 1e-3) / 1e12
    kernels = {k: dict(launches_per_step=v[0] / args.steps, ms_per_step=v[1] / args.steps) for k, v in prof.items()}
    tot_k = sum(v["ms_per_step"] for v in kernels.values()) or 1.0
    for v in kernels.values():
        v["share"] = v["ms_per_step"] / tot_k
    dominant = max(kernels, key=lambda k: kernels[k]["ms_per_step"]) if kernels else None
    roof = dict(bound="hbm", kernel="kda_chunk_fwd (all launches of one call)", achieved=achieved_gbs,
                peak=peaks["hbm_gbs"], unit="GB/s", frac=achieved_gbs / peaks["hbm_gbs"],
                traffic=recorded_traffic("kda_chunk_fwd", th), peak_source=peaks["source"],
                algorithmic_bytes_per_launch=bytes_call, dominant_kernel=dominant,
                intra_tensor_pipe=recorded_tensor_pipe("intra_kernel"))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": ws_n * B, "seq_len": T, "heads": H,
                   "parallelism": f"dp{ws_n} (independent sequences per rank, no collective)",
                   "l2": "inputs larger than L2 (q,k,v,log_alpha,gate,beta = 336 MB per step)"},
        "prefill_tflops": tflops, "prefill_tensor_frac": tflops / peaks["bf16_tflops_sustained"],
        "roofline": roof, "kernels": kernels, "decode": dec, "e2e": e2e, "segment_parallel": seg,
        "kcp_per_device": kcp, "backward": bwd, "varlen": varlen, "long_context": long_ctx,
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": clocks,
    }
    if ws_n == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    return line


def run_decode(args, torch, kda, dev, stream, rank, max_over_ranks, barrier):
    from linear_attention_recurrence_06_b200 import synth
    Bd, H, nsteps, pool = DECODE["Bd"], DECODE["H"], DECODE["steps"], DECODE["pool"]
    state = torch.from_numpy(synth.states(100 + rank, Bd, H, D, D)).to(dev)
    toks = []
    for p in range(pool):
        tb = synth.tokens(200 + rank, p * Bd, Bd, H, D, D, bf16=True)
        toks.append({n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).to(dev)
                     for n in ("q", "k", "v", "log_alpha", "beta")})
    o = torch.empty((Bd, H, D), dtype=torch.bfloat16, device=dev)

    def dstep(i):
        t = toks[i % pool]
        kda.decode_step(state, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], out=o, stream=stream)

    for i in range(3):
        dstep(i)
    torch.cuda.synchronize()
    kda.profile_enable(True)
    for i in range(10):
        dstep(i)
    torch.cuda.synchronize()
    prof = kda.profile_read()
    kda.profile_enable(False)
    kern_ms = prof.get("decode", (10, 0.0))[1] / 10
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(nsteps):
        dstep(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    steps_s = nsteps / (ms * 1e-3)
    state_bytes = DECODE_STATE_BYTES_PER_HEAD * Bd * H
    tok_bytes = DECODE_TOKEN_BYTES_PER_HEAD * Bd * H
    peaks = load_peaks()
    gbs = (state_bytes + tok_bytes) * steps_s / 1e9
    kgbs = (state_bytes + tok_bytes) / (kern_ms * 1e-3) / 1e9 if kern_ms > 0 else None

    # speculative verification: SPEC draft tokens per call (kda_decode_steps), state carried in place
    SPEC = 4
    sq = {n: torch.stack([toks[(i % pool)][n] for i in range(SPEC)]) for n in ("q", "k", "v", "log_alpha", "beta")}
    osp = torch.empty((SPEC, Bd, H, D), dtype=torch.bfloat16, device=dev)

    def vstep():
        kda.decode_steps(state, sq["q"], sq["k"], sq["v"], sq["log_alpha"], sq["beta"], out=osp, stream=stream)

    for _ in range(3):
        vstep()
    ncalls = nsteps // SPEC
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(ncalls):
        vstep()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_v = max_over_ranks(e0.elapsed_time(e1))
    spec = {"draft_tokens_per_call": SPEC, "calls": ncalls, "ms_per_call": ms_v / ncalls,
            "tokens_per_s": ncalls * SPEC / (ms_v * 1e-3),
            "bytes_per_call": state_bytes + SPEC * tok_bytes,
            "gbs": (state_bytes + SPEC * tok_bytes) * ncalls / (ms_v * 1e-3) / 1e9}
    return {"workload": f"KDA decode, {Bd} sequences x {H} heads, fp32 state 128x128 (512 MiB), {nsteps} "
                        f"consecutive steps, bf16 tokens (pool of {pool} distinct steps)",
            "value": steps_s, "unit": "steps/s", "ms_per_step": ms / nsteps, "state_gbs": gbs,
            "hbm_frac": gbs / peaks["hbm_gbs"],
            "roofline": {"bound": "hbm", "kernel": "decode_multi_kernel", "achieved": kgbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": (kgbs / peaks["hbm_gbs"]) if kgbs else None,
                         "traffic": recorded_traffic("decode_multi_kernel", Bd * H),
                         "algorithmic_bytes_per_launch": state_bytes + tok_bytes},
            "speculative_verify": spec}


SEG_SHAPE = dict(T=65536, H=1, segments=32)


def run_segmented(args, torch, kda, dev, stream, max_over_ranks, barrier):
    """One sequence of 65536 tokens, one head (4 chains for the plain walk): the
    plain prefill against the segment-parallel one (32 segments), both with the
    fused gate, decays scaled by 0.01 so that the state carries across segments."""
    from linear_attention_recurrence_06_b200 import synth
    T, H, G = SEG_SHAPE["T"], SEG_SHAPE["H"], SEG_SHAPE["segments"]
    tb = synth.tokens(300, 0, T, H, D, D, bf16=True, gate=True)
    tb.log_alpha = (tb.log_alpha * 0.01).astype(np.float32)
    x = {n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).to(dev)
         for n in ("q", "k", "v", "log_alpha", "beta", "g")}
    x = {n: t.view(1, T, H, -1) if n != "beta" else t.view(1, T, H) for n, t in x.items()}
    out = torch.empty((1, T, H, D), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, H, D, D), dtype=torch.float32, device=dev)
    res = {"workload": f"KDA prefill B=1 T={T} H={H} bf16, fused gate, decays x 0.01", "segments": G}
    for name, segs in (("plain", 1), ("segmented", G)):
        nbytes = kda.segmented_workspace_size(T, H, 1, T, segs) if segs > 1 else kda.workspace_size(T, H, 1, T)[1]
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

        def f():
            kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, gate=x["g"], out=out,
                          final_state=fs, workspace=ws, segments=segs, stream=stream)

        for _ in range(3):
            f()
        n = max(5, min(args.steps, 20))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n):
            f()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms = max_over_ranks(e0.elapsed_time(e1) / n)
        res[name] = {"ms_per_call": ms, "tokens_per_s": T / (ms * 1e-3)}
        del ws
    res["speedup"] = res["plain"]["ms_per_call"] / res["segmented"]["ms_per_call"]
    return res


VARLEN = dict(n_seqs=16, lo=512, hi=16384, H=32)
LONG = dict(T=1 << 20, H=32, pool=65536)
# algorithmic bytes per token-head without the gate: q, k, v, log_alpha in + o out (bf16) + beta
PREFILL_NOGATE_BYTES_PER_TH = 5 * 256 + 2


def _time_calls(torch, f, n, stream, max_over_ranks, barrier):
    for _ in range(3):
        f()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(n):
        f()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(e0.elapsed_time(e1) / n)


def _pool_tokens(torch, dev, seed, n, H):
    """n tokens of every input (bf16, the workload's distributions) on the device."""
    from linear_attention_recurrence_06_b200 import synth
    tb = synth.tokens(seed, 0, n, H, D, D, bf16=True)
    return {k: torch.from_numpy(np.ascontiguousarray(getattr(tb, k))).to(torch.bfloat16).to(dev)
            for k in ("q", "k", "v", "log_alpha", "beta")}


def run_varlen(args, torch, kda, dev, stream, max_over_ranks, barrier):
    """Packed varlen prefill: 16 sequences with lengths uniform on [512, 16384]
    (seeded), H=32, bf16, random fp32 initial states N(0, 0.02^2), final states
    returned.  Token values come from one 16,384-token pool of the same
    distributions (sequence n takes its first L_n tokens): the kernels' time does
    not depend on the values."""
    from linear_attention_recurrence_06_b200 import synth
    n, H = VARLEN["n_seqs"], VARLEN["H"]
    lengths = synth.varlen_lengths(0, n, VARLEN["lo"], VARLEN["hi"])
    cu = synth.cu_from_lengths(lengths)
    T = int(cu[-1])
    pool = _pool_tokens(torch, dev, 500, VARLEN["hi"], H)
    x = {}
    for k, t in pool.items():
        x[k] = torch.cat([t[:int(L)] for L in lengths]).view((1, T, H) + tuple(t.shape[2:]))
    s0 = torch.from_numpy(synth.states(501, n, H, D, D)).to(dev)
    cu_d = torch.from_numpy(cu.astype(np.int32)).to(dev)
    out = torch.empty((1, T, H, D), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((n, H, D, D), dtype=torch.float32, device=dev)
    _, full = kda.workspace_size(T, H, n, int(lengths.max()))
    ws = torch.empty(full, dtype=torch.uint8, device=dev)

    def f():
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], s0, cu_seqlens=cu_d,
                      max_seqlen=int(lengths.max()), out=out, final_state=fs, workspace=ws, stream=stream)

    ms = _time_calls(torch, f, max(5, min(args.steps, 20)), stream, max_over_ranks, barrier)
    th = T * H
    nbytes = PREFILL_NOGATE_BYTES_PER_TH * th + 2 * n * H * D * D * 4
    peaks = load_peaks()
    return {"workload": f"KDA varlen prefill, {n} sequences, lengths uniform on [{VARLEN['lo']}, {VARLEN['hi']}] "
                        f"(seed 0: {T} tokens), H={H}, bf16, fp32 initial and final states",
            "tokens": T, "ms_per_call": ms, "tokens_per_s": T / (ms * 1e-3),
            "algorithmic_bytes": nbytes, "hbm_bound_ms": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3,
            "hbm_frac": nbytes / (ms * 1e-3) / (peaks["hbm_gbs"] * 1e9),
            "tflops": PREFILL_FLOP_PER_TH * th / (ms * 1e-3) / 1e12, "passes": 1}


def run_long(args, torch, kda, dev, stream, max_over_ranks, barrier):
    """Long-context prefill: B=1, T=2^20, H=32, bf16, zero initial state, one pass
    (the whole-sequence workspace).  Token values: a 65,536-token pool of the
    workload's distributions repeated 16 times (timing does not depend on the
    values; the parity test runs fresh tokens throughout)."""
    T, H, P = LONG["T"], LONG["H"], LONG["pool"]
    pool = _pool_tokens(torch, dev, 600, P, H)
    x = {k: t.repeat((T // P,) + (1,) * (t.dim() - 1)).view((1, T, H) + tuple(t.shape[2:])) for k, t in pool.items()}
    del pool
    out = torch.empty((1, T, H, D), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, H, D, D), dtype=torch.float32, device=dev)
    _, full = kda.workspace_size(T, H, 1, T)
    ws = torch.empty(full, dtype=torch.uint8, device=dev)

    def f():
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, out=out, final_state=fs,
                      workspace=ws, stream=stream)

    ms = _time_calls(torch, f, 3, stream, max_over_ranks, barrier)
    th = T * H
    nbytes = PREFILL_NOGATE_BYTES_PER_TH * th
    peaks = load_peaks()
    res = {"workload": f"KDA long-context prefill B=1 T={T} H={H} bf16, zero initial state",
           "tokens": T, "ms_per_call": ms, "tokens_per_s": T / (ms * 1e-3),
           "algorithmic_bytes": nbytes, "hbm_bound_ms": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3,
           "hbm_frac": nbytes / (ms * 1e-3) / (peaks["hbm_gbs"] * 1e9),
           "workspace_bytes": full, "passes": 1,
           "sequential_chunk_steps": T // 64}
    del x, out, ws
    torch.cuda.empty_cache()
    return res


KCP_SHAPE = dict(T_rank=8192, H=32, ranks=8)


# Algorithmic work of the backward per (64-token chunk, head), counted from its products
# (2 FLOP per multiply-add): A and P 4,096 dot products of 128; M^-1 43.7 k; R = V - (K o Gam) S0
# 64x128x128; U, P^T dO, Y (triangular) 3 x 266 k; K^C dS_C 64x128x128; dP, dM 524 k; the three
# (token, channel) accumulations 3 x 64x128x128; the A/P contractions 2 x 524 k.  The reverse
# chain per chunk step and head: M_lr^T dS 128x128x128 and Q'^T dO 128x64x128.
BWD_INTRA_FLOP_PER_ITEM = 2 * (524288 + 43690 + 1048576 + 3 * 266240 + 1048576 + 524288 + 3 * 1048576 + 2 * 524288)
BWD_CHAIN_FLOP_PER_ITEM = 2 * (128 * 128 * 128 + 128 * 64 * 128)
# Tensor-core work the backward kernels issue per (chunk, head) (dense tiles, 2 FLOP per
# multiply-add): the chunk-local kernel's 12 products (stage 1: 128x160x128 + 2 x 128x64x128;
# stage 2: 2 x 128x64x64; stage 3: 128x64x64 + 128x64x128; stage 4: 128x64x128 + 128x128x128;
# stage 5, high and low parts: 2 x 128x128x160 + 2 x 128x160x128); the reverse chain's
# M_lr^T dS and Q'^T dO (as counted above).
BWD_INTRA_ISSUED_FLOP_PER_ITEM = 2 * (128 * 160 * 128 + 2 * 128 * 64 * 128 + 2 * 128 * 64 * 64 + 128 * 64 * 64
                                      + 128 * 64 * 128 + 128 * 64 * 128 + 128 * 128 * 128 + 4 * 128 * 128 * 160)


def run_backward(args, torch, kda, dev, stream, max_over_ranks, barrier):
    """kda_chunk_bwd on the prefill shape (B=1, T=8192, H=32, bf16 inputs and dL/do,
    an initial state and dL/d(final state)): one call = the forward walk recomputed
    without outputs + the reverse walk + the chunk-local gradient kernel."""
    from linear_attention_recurrence_06_b200 import synth
    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    tb = synth.tokens(500, 0, T, H, D, D, bf16=True)
    x = {n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).to(dev)
         for n in ("q", "k", "v", "log_alpha", "beta")}
    x = {n: t.view(1, T, H, -1) if n != "beta" else t.view(1, T, H) for n, t in x.items()}
    d_o = torch.from_numpy(synth.normal(501, synth.TAG_V, (T, H, D), 1.0, True)).to(torch.bfloat16).to(dev)
    d_o = d_o.view(1, T, H, D)
    s0 = torch.from_numpy(synth.states(502, 1, H, D, D)).to(dev)
    dfin = torch.from_numpy(synth.states(503, 1, H, D, D)).to(dev)
    ws = torch.empty(kda.bwd_workspace_size(T, H, 1, T), dtype=torch.uint8, device=dev)

    def f():
        kda.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o, s0, dfin, scale=D ** -0.5,
                      workspace=ws, stream=stream)

    for _ in range(3):
        f()
    n = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(n):
        f()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / n)
    # per-kernel split from a separate, profiled set of calls
    kda.profile_enable(True)
    kda.profile_read()
    for _ in range(n):
        f()
    torch.cuda.synchronize()
    prof = kda.profile_read()
    kda.profile_enable(False)
    kernels = {k: dict(launches_per_call=v[0] / n, ms_per_call=v[1] / n) for k, v in prof.items()}
    # both backward kernels run their products on the tensor cores: roofline against the bf16
    # tensor peak (the sustained figure: the kernels run inside a loop of calls)
    peaks = load_peaks()
    items = B * (T // 64) * H
    roof = {}
    for name, flop, issued in (("intra_bwd", BWD_INTRA_FLOP_PER_ITEM, BWD_INTRA_ISSUED_FLOP_PER_ITEM),
                               ("chain_bwd", BWD_CHAIN_FLOP_PER_ITEM, BWD_CHAIN_FLOP_PER_ITEM)):
        if name in kernels and kernels[name]["ms_per_call"] > 0:
            tf = flop * items / (kernels[name]["ms_per_call"] * 1e-3) / 1e12
            roof[name] = dict(bound="tensor", achieved=tf, peak=peaks["bf16_tflops_sustained"], unit="TFLOP/s",
                              frac=tf / peaks["bf16_tflops_sustained"], flop_per_launch=flop * items,
                              issued_flop_per_launch=issued * items, peak_source=peaks["source"])
    return {"workload": f"KDA backward B={B} T={T} H={H} bf16 inputs and dL/do, fp32 gradients, initial state "
                        "and final-state gradient", "ms_per_call": ms, "tokens_per_s": B * T / (ms * 1e-3),
            "kernels": kernels, "roofline": roof}


def run_kcp(args, torch, kda, dev, stream, max_over_ranks, barrier):
    """The work one device does when a sequence of ranks x 8192 tokens (32 heads,
    fused gate) is split over `ranks` devices: transition (chunk-local kernel +
    the walk that forms M and B), compose of the maps of all earlier devices
    (the last device's case: ranks - 1 maps) and finish (the walk with outputs),
    next to the plain prefill of the same 8192 tokens.  The all-gather between
    transition and compose is not timed (one GPU); its size is reported."""
    from linear_attention_recurrence_06_b200 import synth
    T, H, R = KCP_SHAPE["T_rank"], KCP_SHAPE["H"], KCP_SHAPE["ranks"]
    tb = synth.tokens(400, 0, T, H, D, D, bf16=True, gate=True)
    x = {n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).to(dev)
         for n in ("q", "k", "v", "log_alpha", "beta", "g")}
    x = {n: t.view(1, T, H, -1) if n != "beta" else t.view(1, T, H) for n, t in x.items()}
    out = torch.empty((1, T, H, D), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(kda.kcp_workspace_size(T, H, 1, T), dtype=torch.uint8, device=dev)
    trans = torch.empty((2, 1, H, D, D), dtype=torch.float32, device=dev)
    s_in = torch.empty((1, H, D, D), dtype=torch.float32, device=dev)
    s0 = torch.zeros((1, H, D, D), dtype=torch.float32, device=dev)
    steps = {
        "transition": lambda: kda.kcp_transition(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                                 transition=trans, workspace=ws, stream=stream),
        "compose": lambda: kda.kcp_compose(gathered, R - 1, s0, out=s_in, stream=stream),
        "finish": lambda: kda.kcp_finish(s_in, ws, shape=(1, T, H, D), dtype=torch.bfloat16, gate=x["g"],
                                         out=out, stream=stream),
        "plain": lambda: kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, gate=x["g"],
                                       out=out, final_state=fs, workspace=ws, stream=stream),
    }
    steps["transition"]()
    torch.cuda.synchronize()
    gathered = trans.unsqueeze(0).expand((R,) + tuple(trans.shape)).contiguous()  # stands for the all-gather
    res = {"workload": f"one sequence of {R} x {T} tokens, H={H}, bf16, fused gate; per device",
           "ranks": R, "tokens_per_device": T,
           "all_gather_bytes_per_device": trans.numel() * trans.element_size()}
    # order matters: finish reads the slots transition left in the workspace
    for name in ("transition", "compose", "finish", "plain"):
        f = steps[name]
        for _ in range(3):
            f()
        n = max(5, min(args.steps, 20))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n):
            f()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        res[name + "_ms"] = max_over_ranks(e0.elapsed_time(e1) / n)
    res["device_ms"] = res["transition_ms"] + res["compose_ms"] + res["finish_ms"]
    res["overhead_vs_plain"] = res["device_ms"] / res["plain_ms"]
    res["sequence_tokens_per_s_without_gather"] = R * T / (res["device_ms"] * 1e-3)
    return res


def run_kcp_ranks(args, torch, kda, dev, stream, rank, world, max_over_ranks, barrier):
    """One sequence of world x 8192 tokens (32 heads, fused gate) split over the ranks of
    this job: every rank runs kcp.kcp_prefill on its segment (transition, NCCL all-gather
    of the 4 MiB of segment maps, compose, finish).  Time = max over ranks."""
    from linear_attention_recurrence_06_b200 import kcp, synth
    T, H = KCP_SHAPE["T_rank"], KCP_SHAPE["H"]
    tb = synth.tokens(400, rank * T, T, H, D, D, bf16=True, gate=True)
    x = {n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).to(dev)
         for n in ("q", "k", "v", "log_alpha", "beta", "g")}
    x = {n: t.view(1, T, H, -1) if n != "beta" else t.view(1, T, H) for n, t in x.items()}

    def f():
        return kcp.kcp_prefill(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, gate=x["g"],
                               stream=stream)

    for _ in range(3):
        f()
    n = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(n):
        f()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / n)
    return {"ranks": world, "tokens_per_rank": T, "ms_per_call": ms,
            "sequence_tokens_per_s": world * T / (ms * 1e-3),
            "all_gather_bytes_per_rank": 2 * H * D * D * 4}


def run_e2e(args, torch, kda, hq, out, fs, ws, stream, max_over_ranks, barrier):
    """End to end through the public API: every step copies its inputs from
    pinned host memory, runs kda_chunk_fwd and reads its output back to pinned
    host memory.  Consecutive steps are pipelined over two device buffer sets:
    step i+1's host->device copy (copy stream) and step i-1's device->host read
    (read-back stream) overlap step i's compute (PCIe is full duplex)."""
    B, T, H = PREFILL["B"], PREFILL["T"], PREFILL["H"]
    dev = out.device
    sets = [{n: torch.empty_like(t, device=dev) for n, t in hq.items()} for _ in range(2)]
    outs = [out, torch.empty_like(out)]
    houts = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hq.values())
    d2h = houts[0].numel() * houts[0].element_size()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    in_ready, computed, read_back = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def estep(i):
        j = i & 1
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(computed[j])  # set j's inputs are no longer read
            for n in hq:
                sets[j][n].copy_(hq[n], non_blocking=True)
            in_ready[j].record(s_in)
        stream.wait_event(in_ready[j])
        if used[j]:
            stream.wait_event(read_back[j])  # set j's output was read back
        d = sets[j]
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, gate=d["g"], out=outs[j],
                      final_state=fs, workspace=ws, stream=stream)
        computed[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[j])
            houts[j].copy_(outs[j], non_blocking=True)
            read_back[j].record(s_out)
        used[j] = True

    for i in range(2):
        estep(i)
    torch.cuda.synchronize()
    n = max(4, min(args.steps, 12))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(n):
        estep(i)
    stream.wait_stream(s_out)  # the last read-back is inside the timed region
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / n)
    ws_n = int(os.environ.get("WORLD_SIZE", "1"))
    return {"value": whole_job_rate(ws_n, B * T, ms), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "two buffer sets; copy-in, compute and read-back of consecutive steps overlap"}


def recorded_tensor_pipe(kernel: str):
    """Tensor-pipe activity of a kernel from the committed ncu summary (fraction of its
    elapsed cycles, and over its tensor-core product stages), if taken on the current
    sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rec = json.load(open(p)).get(kernel)
    except Exception:
        return None
    if not rec or rec.get("sources_sha256") != sources_sha256(kernel) or "tensor_pipe_active_frac" not in rec:
        return None
    return {"active_frac": rec["tensor_pipe_active_frac"],
            "active_frac_over_product_stages": rec.get("tensor_pipe_active_frac_over_product_stages"),
            "source": "ncu sm__pipe_tensor_cycles_active, profiles/kda_intra_T4096_H32_ncu_full.md"}


def recorded_traffic(kernel: str, units: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rec = json.load(open(p)).get(kernel)
    except Exception:
        return None
    if not rec or rec.get("sources_sha256") != sources_sha256(kernel):
        return None
    return rec["dram_bytes_per_unit"] * units


# the source files each recorded kernel is built from (a change to any of them
# voids its recorded traffic)
KERNEL_SOURCES = {
    "kda_chunk_fwd": ("kda_chunk.cu", "kda_sm100.cuh", "kda_slots.h", "kda_tri.cuh"),
    "intra_kernel": ("kda_chunk.cu", "kda_sm100.cuh", "kda_slots.h", "kda_tri.cuh"),
    "chain_kernel": ("kda_chunk.cu", "kda_sm100.cuh", "kda_slots.h"),
    "decode_multi_kernel": ("kda_decode.cu", "kda_sm100.cuh"),
    "bwd_tc_kernel": ("kda_bwd.cu", "kda_sm100.cuh", "kda_slots.h", "kda_tri.cuh"),
    "chain_bwd_tc_kernel": ("kda_bwd.cu", "kda_sm100.cuh", "kda_slots.h"),
}


def sources_sha256(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_recurrence_06_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()


# ------------------------------------------------------------- CPU baseline

def oracle_sample_rate(n_tokens: int, heads: int, threads: int = 0):
    """Runs the fp64 oracle (recurrence + gate-norm) on the first n_tokens of
    the prefill workload for `heads` heads; returns (seconds, threads used)."""
    import oracle
    from linear_attention_recurrence_06_b200 import synth
    H = PREFILL["H"]
    tb = synth.tokens(0, 0, n_tokens, H, D, D, bf16=True, gate=True)
    t0 = time.perf_counter()
    o, _, nt = oracle.kda_recurrent(tb.q, tb.k, tb.v, tb.log_alpha, tb.beta, heads=(0, heads), n_threads=threads,
                                    return_threads=True)
    oracle.gate_norm(o[:, :heads], tb.g[:, :heads], None, 1e-6)
    return time.perf_counter() - t0, nt


def cpu_baseline(seconds: float = 10.0):
    import oracle
    H = PREFILL["H"]
    cores = oracle.available_cores()
    probe_tokens = 64
    dt, _ = oracle_sample_rate(probe_tokens, H)
    n_tok = int(min(PREFILL["T"], max(probe_tokens, probe_tokens * seconds / max(dt, 1e-6))))
    dt, nt = oracle_sample_rate(n_tok, H)
    return {"value": n_tok / dt, "unit": "tokens/s", "cores": nt, "kind": "oracle",
            "sample": f"first {n_tok} of {PREFILL['T']} tokens, all {H} heads, fp64 recurrence + gate-norm, "
                      f"{dt:.1f} s on {nt} threads ({cores} cores available)"}


# -------------------------------------------------------- reference arm (oracle)

def run_reference(args):
    ws_n, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    H = PREFILL["H"]
    n_tok = args.ref_tokens
    for _ in range(args.warmup):
        oracle_sample_rate(n_tok, H)
    times, nt = [], 1
    for _ in range(args.steps):
        dt, nt = oracle_sample_rate(n_tok, H)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = n_tok / (ms * 1e-3)
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": PREFILL["T"], "heads": H,
                       "parallelism": "host threads over (sequence, head)", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nt, "kind": "oracle",
                             "sample": f"each step: first {n_tok} of {PREFILL['T']} tokens, all {H} heads"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_ncu_decode_case(args):
    """Decode case for profiler captures: `warmup + steps` single decode steps on
    the 256 x 32 workload (512 MiB fp32 state), no timing."""
    import torch
    import linear_attention_recurrence_06_b200 as kda
    from linear_attention_recurrence_06_b200 import synth
    Bd, H = DECODE["Bd"], DECODE["H"]
    state = torch.from_numpy(synth.states(100, Bd, H, D, D)).cuda()
    tb = synth.tokens(200, 0, Bd, H, D, D, bf16=True)
    t = {n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).cuda()
         for n in ("q", "k", "v", "log_alpha", "beta")}
    o = torch.empty((Bd, H, D), dtype=torch.bfloat16, device="cuda")
    for _ in range(args.warmup + args.steps):
        kda.decode_step(state, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], out=o)
    torch.cuda.synchronize()
    return {"ncu_case": f"decode Bd={Bd} H={H}", "calls": args.warmup + args.steps}


def run_ncu_case(args):
    """Small prefill case for profiler captures: `warmup + steps` calls of
    kda_chunk_fwd (fused gate) on T = --ncu-tokens tokens, H = 32, no timing."""
    import torch
    import linear_attention_recurrence_06_b200 as kda
    from linear_attention_recurrence_06_b200 import synth
    T, H = args.ncu_tokens, PREFILL["H"]
    tb = synth.tokens(0, 0, T, H, D, D, bf16=True, gate=True)
    up = {n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).cuda()
          for n in ("q", "k", "v", "log_alpha", "beta", "g")}
    x = {n: t.view(1, T, H, -1) if n != "beta" else t.view(1, T, H) for n, t in up.items()}
    out = torch.empty((1, T, H, D), dtype=torch.bfloat16, device="cuda")
    fs = torch.empty((1, H, D, D), dtype=torch.float32, device="cuda")
    _, full = kda.workspace_size(T, H, 1, T)
    ws = torch.empty(full, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup + args.steps):
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, gate=x["g"], out=out,
                      final_state=fs, workspace=ws)
    torch.cuda.synchronize()
    return {"ncu_case": f"prefill T={T} H={H}", "calls": args.warmup + args.steps, "status": kda.query_status(ws)}


def run_ncu_bwd_case(args):
    """Small backward case for profiler captures: `warmup + steps` calls of kda_chunk_bwd
    on T = --ncu-bwd-tokens tokens, H = 32, bf16 inputs and dL/do, no timing."""
    import torch
    import linear_attention_recurrence_06_b200 as kda
    from linear_attention_recurrence_06_b200 import synth
    T, H = args.ncu_bwd_tokens, PREFILL["H"]
    tb = synth.tokens(500, 0, T, H, D, D, bf16=True)
    up = {n: torch.from_numpy(np.ascontiguousarray(getattr(tb, n))).to(torch.bfloat16).cuda()
          for n in ("q", "k", "v", "log_alpha", "beta")}
    x = {n: t.view(1, T, H, -1) if n != "beta" else t.view(1, T, H) for n, t in up.items()}
    d_o = torch.from_numpy(synth.normal(501, synth.TAG_V, (T, H, D), 1.0, True)).to(torch.bfloat16).cuda()
    ws = torch.empty(kda.bwd_workspace_size(T, H, 1, T), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup + args.steps):
        kda.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o.view(1, T, H, D), None, None,
                      scale=D ** -0.5, workspace=ws)
    torch.cuda.synchronize()
    return {"ncu_case": f"backward T={T} H={H}", "calls": args.warmup + args.steps, "status": kda.query_status(ws)}


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def launch_ranks(n: int, argv) -> int:
    """Re-runs this script as n ranks of one node (torch.distributed.run, one
    process per GPU, rendezvous on 127.0.0.1).  The ranks' output passes through;
    rank 0 prints the JSON line.  Returns the launcher's exit code."""
    env = dict(os.environ)
    # NCCL prints its communicator set-up (ranks, transport) so the rank count is on record
    env.setdefault("NCCL_DEBUG", "INFO")
    env.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    return subprocess.run(cmd, env=env).returncode


def run_dry(args):
    """The multi-rank plumbing without a GPU: every rank joins a gloo process
    group, reports its rank and takes part in the max-over-ranks reduction that
    the timed runs use; rank 0 prints what it saw."""
    import datetime
    import torch
    import torch.distributed as dist
    ws_n, rank, _ = dist_env()
    if ws_n > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    ranks = torch.zeros(ws_n, dtype=torch.float64)
    ranks[rank] = 1.0
    if ws_n > 1:
        dist.all_reduce(ranks)
    ms = max_over_ranks(float(rank + 1), dist if ws_n > 1 else None)
    if ws_n > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    return {"dry_run": True, "n_gpus": ws_n, "ranks_reported": int(ranks.sum().item()), "max_over_ranks": ms,
            "value": whole_job_rate(ws_n, 1.0, ms)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-tokens", type=int, default=256)
    ap.add_argument("--ncu-tokens", type=int, default=0,
                    help="profiler case: only run warmup+steps prefill calls on this many tokens")
    ap.add_argument("--ncu-bwd-tokens", type=int, default=0,
                    help="profiler case: only run warmup+steps backward calls on this many tokens")
    ap.add_argument("--ncu-decode", action="store_true",
                    help="profiler case: only run warmup+steps decode steps on the 256 x 32 workload")
    ap.add_argument("--dry-run", action="store_true",
                    help="no GPU work: ranks join a gloo group and report (tests the multi-rank launch)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws_env = os.environ.get("WORLD_SIZE")
    if args.gpus > 1 and ws_env is None:
        # not launched by torch.distributed.run: start one rank per GPU here
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    if ws_env is not None and int(ws_env) != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={ws_env}: launch one rank per GPU")
    if args.dry_run:
        line = run_dry(args)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    peaks = load_peaks()
    if args.ncu_decode:
        line = run_ncu_decode_case(args)
    elif args.ncu_tokens > 0:
        line = run_ncu_case(args)
    elif args.ncu_bwd_tokens > 0:
        line = run_ncu_bwd_case(args)
    else:
        line = run_reference(args) if args.impl == "reference" else run_ours(args, peaks)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
