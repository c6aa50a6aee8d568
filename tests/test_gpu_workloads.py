"""Parity at the full workload sizes, in the launch configuration bench.py times.

The CUDA path runs every head; the fp64 oracle recomputes a sample of heads
(first, a middle one and last) over every token, and the outputs / final states of those
heads are compared element by element (relative L2 <= 1e-2).

  * prefill  B=1, T=8192, H=32, bf16, fused RMSNorm + sigmoid gate
  * varlen   16 sequences, lengths uniform on [512, 16384], H=32, bf16,
             random initial states N(0, 0.02^2), final states returned
  * decode   256 sequences x 32 heads, fp32 state N(0, 0.02^2), 1000
             consecutive steps with fresh bf16 tokens
  * long     B=1, T=2^20, H=32, bf16 (multi-pass workspace), then 64 decode
             steps from the final state
"""
import numpy as np
import pytest

import oracle
from kda_testutil import REL_L2_TOL, D, assert_rel_l2, rel_l2
from linear_attention_recurrence_06_b200 import synth

pytestmark = pytest.mark.gpu

SAMPLE_HEADS = (0, 17, 31)
H = 32


def _t():
    import torch
    return torch


def upload_tokens(torch, T, seed, gate, block=8192):
    """Device bf16 tensors [1, T, H, D] (+ beta [1, T, H]) generated block by
    block; returns them with float32 host copies of the sampled heads."""
    dev = {n: torch.empty((1, T, H, D), dtype=torch.bfloat16, device="cuda")
           for n in ("q", "k", "v", "log_alpha") + (("g",) if gate else ())}
    dev["beta"] = torch.empty((1, T, H), dtype=torch.bfloat16, device="cuda")
    hs = list(SAMPLE_HEADS)
    host = {n: np.empty((T, len(hs), D), np.float32) for n in dev if n != "beta"}
    host["beta"] = np.empty((T, len(hs)), np.float32)
    for t0 in range(0, T, block):
        n = min(block, T - t0)
        tb = synth.tokens(seed, t0, n, H, D, D, bf16=True, gate=gate)
        for name in dev:
            arr = getattr(tb, name)
            dev[name][0, t0:t0 + n].copy_(torch.from_numpy(arr).to(torch.bfloat16))
            host[name][t0:t0 + n] = arr[:, hs]
    return dev, host


def oracle_heads(host, s0=None, cu=None, gate=False):
    """Oracle over the sampled heads only (they are the head axis of `host`)."""
    o, fs = oracle.kda_recurrent(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], s0, cu)
    if gate:
        o = oracle.gate_norm(o, host["g"], None, 1e-6)
    return o, fs


def test_prefill_T8192_H32_gate():
    torch = _t()
    import linear_attention_recurrence_06_b200 as kda
    T = 8192
    dev, host = upload_tokens(torch, T, seed=0, gate=True)
    y, fs = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], None, gate=dev["g"])
    torch.cuda.synchronize()
    ry, rfs = oracle_heads(host, gate=True)
    hs = list(SAMPLE_HEADS)
    yh = y[0][:, hs].float().cpu().numpy()
    fh = fs[0, hs].cpu().numpy()
    assert_rel_l2(yh, ry, "y, sampled heads")
    assert_rel_l2(fh, rfs[0], "final state, sampled heads")


def test_varlen_16_sequences():
    torch = _t()
    import linear_attention_recurrence_06_b200 as kda
    lengths = synth.varlen_lengths(0, 16, 512, 16384)
    cu = synth.cu_from_lengths(lengths)
    T = int(cu[-1])
    dev, host = upload_tokens(torch, T, seed=2, gate=False)
    s0 = synth.states(2, 16, H, D, D)
    hs = list(SAMPLE_HEADS)
    o, fs = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                          torch.from_numpy(s0).cuda(), cu_seqlens=torch.from_numpy(cu.astype(np.int32)).cuda(),
                          max_seqlen=int(lengths.max()))
    torch.cuda.synchronize()
    ro, rfs = oracle_heads(host, s0=s0[:, hs], cu=cu)
    oh = o[0][:, hs].float().cpu().numpy()
    fh = fs[:, hs].cpu().numpy()
    assert_rel_l2(oh, ro, "o, sampled heads")
    assert_rel_l2(fh, rfs, "final states, sampled heads")
    for n in range(16):  # every sequence on its own
        sl = slice(cu[n], cu[n + 1])
        assert_rel_l2(oh[sl], ro[sl], f"seq {n} o")
        assert_rel_l2(fh[n], rfs[n], f"seq {n} final state")


def test_decode_256x32_1000_steps():
    torch = _t()
    import linear_attention_recurrence_06_b200 as kda
    Bd, steps = 256, 1000
    hs = list(SAMPLE_HEADS)
    s_np = synth.states(3, Bd, H, D, D)
    state = torch.from_numpy(s_np).cuda()
    ref = s_np[:, hs].astype(np.float64)
    worst = 0.0
    for step in range(steps):
        tb = synth.tokens(3, step * Bd, Bd, H, D, D, bf16=True)
        args = [torch.from_numpy(getattr(tb, n)).to(torch.bfloat16).cuda() for n in ("q", "k", "v", "log_alpha", "beta")]
        o = kda.decode_step(state, *args)
        ro, ref = oracle.decode_steps(ref, tb.q[:, hs], tb.k[:, hs], tb.v[:, hs], tb.log_alpha[:, hs], tb.beta[:, hs])
        if step % 50 == 0 or step == steps - 1:
            torch.cuda.synchronize()
            e = assert_rel_l2(o[:, hs].float().cpu().numpy(), ro, f"step {step} o")
            worst = max(worst, e)
    torch.cuda.synchronize()
    assert_rel_l2(state[:, hs].cpu().numpy(), ref, "state after 1000 steps")


def test_long_context_1M_then_64_decode_steps():
    torch = _t()
    import linear_attention_recurrence_06_b200 as kda
    T = 1 << 20
    hs = list(SAMPLE_HEADS)
    dev, host = upload_tokens(torch, T, seed=4, gate=False)
    lo, _ = kda.workspace_size(T, H, 1, T)
    ws = torch.empty(max(lo, 2 << 30), dtype=torch.uint8, device="cuda")  # many passes
    o, fs = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], None, workspace=ws)
    torch.cuda.synchronize()
    assert kda.query_status(ws) == 0
    ro, rfs = oracle_heads(host)
    oh = o[0][:, hs].float().cpu().numpy()
    assert_rel_l2(oh, ro, "o, sampled heads")
    # the last 64 Ki tokens on their own (late-sequence accuracy)
    assert_rel_l2(oh[-65536:], ro[-65536:], "o, last 64 Ki tokens")
    assert_rel_l2(fs[0, hs].cpu().numpy(), rfs[0], "final state")
    del dev, o
    # 64 decode steps continue from the prefill's final state
    state = fs.clone()
    ref = rfs[:, :].copy()
    for step in range(64):
        tb = synth.tokens(5, step, 1, H, D, D, bf16=True)
        args = [torch.from_numpy(getattr(tb, n)).to(torch.bfloat16).cuda() for n in ("q", "k", "v", "log_alpha", "beta")]
        od = kda.decode_step(state, *args, out_dtype=torch.float32)
        rod, ref = oracle.decode_steps(ref, tb.q[:, hs], tb.k[:, hs], tb.v[:, hs], tb.log_alpha[:, hs], tb.beta[:, hs])
        torch.cuda.synchronize()
        assert_rel_l2(od[:, hs].cpu().numpy(), rod, f"decode step {step} o")
    assert_rel_l2(state[:, hs].cpu().numpy(), ref, "state after 64 decode steps")
