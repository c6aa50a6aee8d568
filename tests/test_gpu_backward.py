"""GPU parity of the backward pass (kda_chunk_bwd, through the C ABI binding)
against the fp64 oracle's exact gradients (oracle.kda_recurrent_bwd) on the
same seeded inputs and output gradients: relative L2 <= 1e-2 per gradient."""
import numpy as np
import pytest

import oracle
from kda_testutil import REL_L2_TOL, D, dev, host, make_prefill, rel_l2
from linear_attention_recurrence_06_b200 import synth

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


def _grads_case(seed, lens, H, bf16=True, init=True, d_final=True, scale=0.125, **kw):
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    inp = make_prefill(seed, lens, H, bf16=bf16, init=init, **kw)
    T = inp["T"]
    dt = torch.bfloat16 if bf16 else torch.float32
    d_o = synth.normal(seed + 1000, synth.TAG_V, (T, H, D), 1.0, bf16)
    d_fin = synth.states(seed + 2000, len(lens), H, D, D, std=0.5) if d_final else None
    q, k, v, la = (dev(inp[x], dt).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha"))
    b = dev(inp["beta"], dt).view(1, T, H)
    do_t = dev(d_o, dt).view(1, T, H, D)
    s0 = dev(inp["s0"], torch.float32) if init else None
    dfin = dev(d_fin, torch.float32) if d_final else None
    cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
    g = kda.chunk_bwd(q, k, v, la, b, do_t, s0, dfin, cu_seqlens=cu, max_seqlen=max(max(lens), 0), scale=scale)
    torch.cuda.synchronize()
    ref = oracle.kda_recurrent_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o, inp["s0"],
                                   d_fin, inp["cu"], scale=scale)
    mine = {
        "dq": host(g["dq"]).reshape(T, H, D), "dk": host(g["dk"]).reshape(T, H, D),
        "dv": host(g["dv"]).reshape(T, H, D), "dlog_alpha": host(g["dlog_alpha"]).reshape(T, H, D),
        "dbeta": host(g["dbeta"]).reshape(T, H), "d_init": host(g["d_initial_state"]),
    }
    return mine, ref, inp


def _check(mine, ref, what=""):
    errs = {k: rel_l2(mine[k], ref[k]) for k in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_init")}
    bad = {k: e for k, e in errs.items() if not e <= REL_L2_TOL}
    assert not bad, f"{what} rel-L2 above {REL_L2_TOL}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("lens,H,bf16", [
    ([200], 2, True),
    ([64], 1, True),
    ([1, 15, 16, 17, 63, 64, 65, 0, 130], 2, True),
    ([150], 3, False),
])
def test_backward_matches_oracle(lens, H, bf16):
    mine, ref, _ = _grads_case(81 + len(lens), lens, H, bf16=bf16)
    _check(mine, ref, f"lens={lens}")


@pytest.mark.parametrize("case", ["long_memory", "clamped", "no_state_terms"])
def test_backward_regimes(case):
    """Long memory (decays x 0.01: the state carries across chunks), many
    log-decays below the floor (the clamp blocks their gradient), and no initial
    state / no final-state gradient."""
    kw = dict(long_memory=dict(la_scale=0.01), clamped=dict(la_scale=8.0), no_state_terms={})[case]
    extra = dict(init=False, d_final=False) if case == "no_state_terms" else {}
    mine, ref, inp = _grads_case(91, [333, 70], 2, **kw, **extra)
    _check(mine, ref, case)
    if case == "clamped":
        below = inp["log_alpha"] < -5.0
        assert below.any()
        assert np.all(mine["dlog_alpha"][below] == 0.0)


def test_backward_per_sequence_and_token_tail():
    """Worst sequence and the last chunk's tokens on their own (a ragged tail)."""
    lens = [300, 129, 64, 5]
    mine, ref, inp = _grads_case(97, lens, 2)
    for n, L in enumerate(lens):
        sl = slice(inp["cu"][n], inp["cu"][n + 1])
        for k in ("dq", "dk", "dv", "dlog_alpha"):
            assert rel_l2(mine[k][sl], ref[k][sl]) <= REL_L2_TOL, f"seq {n} {k}"
        tail = slice(inp["cu"][n] + (L - 1) // 64 * 64, inp["cu"][n + 1])
        assert rel_l2(mine["dk"][tail], ref["dk"][tail]) <= REL_L2_TOL, f"seq {n} tail dk"
        assert rel_l2(mine["d_init"][n], ref["d_init"][n]) <= REL_L2_TOL, f"seq {n} d_init"


def test_backward_fixed_length_batch():
    """B = 2 sequences of 100 tokens without cu_seqlens ([B, T, H, 128] layout)."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    B, T, H = 2, 100, 2
    inp = make_prefill(99, [T] * B, H, bf16=True, init=True)
    dt = torch.bfloat16
    d_o = synth.normal(1099, synth.TAG_V, (B * T, H, D), 1.0, True)
    d_fin = synth.states(2099, B, H, D, D, std=0.5)
    q, k, v, la = (dev(inp[x], dt).view(B, T, H, D) for x in ("q", "k", "v", "log_alpha"))
    b = dev(inp["beta"], dt).view(B, T, H)
    g = kda.chunk_bwd(q, k, v, la, b, dev(d_o, dt).view(B, T, H, D), dev(inp["s0"], torch.float32),
                      dev(d_fin, torch.float32), scale=0.2)
    torch.cuda.synchronize()
    ref = oracle.kda_recurrent_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o, inp["s0"],
                                   d_fin, inp["cu"], scale=0.2)
    mine = {"dq": host(g["dq"]).reshape(B * T, H, D), "dk": host(g["dk"]).reshape(B * T, H, D),
            "dv": host(g["dv"]).reshape(B * T, H, D), "dlog_alpha": host(g["dlog_alpha"]).reshape(B * T, H, D),
            "dbeta": host(g["dbeta"]).reshape(B * T, H), "d_init": host(g["d_initial_state"])}
    _check(mine, ref, "B=2 fixed length")
