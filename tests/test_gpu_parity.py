"""GPU parity: the CUDA path (through the C ABI binding) against the fp64 oracle
on the same seeded inputs, element by element, relative L2 <= 1e-2."""
import numpy as np
import pytest

import oracle
from kda_testutil import REL_L2_TOL, D, assert_rel_l2, dev, guarded_empty, host, make_prefill, rel_l2
from linear_attention_recurrence_06_b200 import synth

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


def run_prefill(inp, H, bf16, *, varlen, gate=False, out_f32=False, scale=1.0):
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    dt = torch.bfloat16 if bf16 else torch.float32
    T = inp["T"]
    q = dev(inp["q"], dt).view(1, T, H, D)
    k = dev(inp["k"], dt).view(1, T, H, D)
    v = dev(inp["v"], dt).view(1, T, H, D)
    la = dev(inp["log_alpha"], dt).view(1, T, H, D)
    b = dev(inp["beta"], dt).view(1, T, H)
    g = dev(inp["g"], dt).view(1, T, H, D) if gate else None
    s0 = dev(inp["s0"], torch.float32) if inp["s0"] is not None else None
    kw = {}
    if varlen:
        kw = dict(cu_seqlens=torch.from_numpy(inp["cu"].astype(np.int32)).cuda(),
                  max_seqlen=int(np.diff(inp["cu"]).max()))
    # outputs inside canary guard regions (checked after the call)
    N = len(inp["cu"]) - 1 if varlen else 1
    o, o_check = guarded_empty((1, T, H, D), torch.float32 if out_f32 else dt)
    fs, fs_check = guarded_empty((N, H, D, D), torch.float32)
    kda.chunk_fwd(q, k, v, la, b, s0, gate=g, scale=scale, out=o, final_state=fs, **kw)
    o_check("o")
    fs_check("final state")
    return host(o).reshape(T, H, D), host(fs)


def oracle_prefill(inp, gate=False, scale=1.0):
    o, fs = oracle.kda_recurrent(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["s0"], inp["cu"],
                                 scale=scale)
    if gate:
        o = oracle.gate_norm(o, inp["g"], None, 1e-6)
    return o, fs


def check(o, fs, ro, rfs, what=""):
    eo = assert_rel_l2(o, ro, f"{what} output".strip())
    ef = assert_rel_l2(fs, rfs, f"{what} final state".strip())
    return eo, ef


# ----------------------------------------------------------------- prefill


def test_prefill_fp32_small_config():
    """T=256, H=2, fp32 inputs and output, zero initial state, seed 0."""
    inp = make_prefill(0, [256], 2, bf16=False)
    o, fs = run_prefill(inp, 2, False, varlen=False)
    ro, rfs = oracle_prefill(inp)
    check(o, fs, ro, rfs)


@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 200, 333])
def test_prefill_ragged_lengths_bf16(T):
    inp = make_prefill(T, [T], 3, bf16=True, init=True)
    o, fs = run_prefill(inp, 3, True, varlen=False, out_f32=True)
    ro, rfs = oracle_prefill(inp)
    check(o, fs, ro, rfs)


def test_prefill_varlen_edge_lengths():
    lens = [1, 15, 16, 17, 63, 64, 65, 0, 130]
    inp = make_prefill(5, lens, 2, bf16=True, init=True)
    o, fs = run_prefill(inp, 2, True, varlen=True, out_f32=True)
    ro, rfs = oracle_prefill(inp)
    check(o, fs, ro, rfs)
    # per sequence, worst case
    for n in range(len(lens)):
        sl = slice(inp["cu"][n], inp["cu"][n + 1])
        if lens[n]:
            assert_rel_l2(o[sl], ro[sl], f"seq {n} o")
        assert_rel_l2(fs[n], rfs[n], f"seq {n} final state")


# Output scales other than 1 (the usual dk^-1/2 among them).  The scale enters
# the chunk's P and Q' terms and the decode output; the gate's RMSNorm is
# invariant to it, so the ungated cases are the ones that see a misplaced factor.
SCALES = (0.125, 128 ** -0.5)


@pytest.mark.parametrize("scale", SCALES)
@pytest.mark.parametrize("bf16,gate,varlen", [
    (True, False, False), (True, True, False), (False, False, False), (False, True, False),
    (True, False, True), (True, True, True), (False, False, True),
])
def test_prefill_scale(scale, bf16, gate, varlen):
    """Prefill with scale != 1 against the oracle with the same scale: bf16
    and fp32 inputs, with and without the gate, one sequence or packed
    sequences (an empty and ragged ones) with initial states."""
    lens = [200, 64, 0, 77] if varlen else [300]
    H = 3
    inp = make_prefill(17 + int(1000 * scale), lens, H, bf16=bf16, gate=gate, init=True)
    o, fs = run_prefill(inp, H, bf16, varlen=varlen, gate=gate, out_f32=True, scale=scale)
    ro, rfs = oracle_prefill(inp, gate=gate, scale=scale)
    check(o, fs, ro, rfs, f"scale={scale:.4f}")
    if not gate:
        # o is linear in the scale: the unscaled oracle times the scale is the same answer
        ro1, _ = oracle_prefill(inp, gate=False, scale=1.0)
        assert_rel_l2(o, scale * ro1, "o against scale x unscaled oracle")
    if varlen:
        for n, L in enumerate(lens):
            sl = slice(inp["cu"][n], inp["cu"][n + 1])
            if L:
                assert_rel_l2(o[sl], ro[sl], f"seq {n} output")


@pytest.mark.parametrize("case", ["la_floor", "la_zero", "beta_zero", "beta_one", "la_below_floor"])
def test_prefill_degenerate_decays(case):
    kw = {}
    if case == "la_floor":
        kw = dict(la_const=-5.0)
    elif case == "la_zero":
        kw = dict(la_const=0.0)
    elif case == "beta_zero":
        # nothing is written; keep the decay mild so the pure-decay state stays
        # inside the fp32 range (e^{-0.8 * 190} would underflow)
        kw = dict(beta_const=0.0, la_scale=0.05)
    elif case == "beta_one":
        kw = dict(beta_const=1.0)
    elif case == "la_below_floor":
        kw = dict(la_scale=8.0)   # many values far below -5: the clamp path
    inp = make_prefill(11, [190], 2, bf16=True, init=True, **kw)
    o, fs = run_prefill(inp, 2, True, varlen=False, out_f32=True)
    ro, rfs = oracle_prefill(inp)
    check(o, fs, ro, rfs)


@pytest.mark.parametrize("out_f32", [False, True])
def test_prefill_fused_gate_norm(out_f32):
    inp = make_prefill(3, [300], 4, bf16=True, gate=True)
    o, fs = run_prefill(inp, 4, True, varlen=False, gate=True, out_f32=out_f32)
    ro, rfs = oracle_prefill(inp, gate=True)
    check(o, fs, ro, rfs)


@pytest.mark.parametrize("bf16", [True, False])
def test_prefill_gate_varlen_weights_multi_pass(bf16):
    """Gate + RMSNorm with per-channel weights on packed sequences (an empty and
    ragged ones included), once with the full workspace and once with one small
    enough to force one pass per chunk.  bf16 inputs take the normalisation
    fused into the chain (row sums exchanged inside a cluster); fp32 inputs
    take the separate row kernel."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    lens = [1, 64, 0, 200, 17, 129]
    H = 3
    inp = make_prefill(21, lens, H, bf16=bf16, gate=True, init=True)
    T = inp["T"]
    dt = torch.bfloat16 if bf16 else torch.float32
    q, k, v, la, g = (dev(inp[x], dt).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha", "g"))
    b = dev(inp["beta"], dt).view(1, T, H)
    s0 = dev(inp["s0"], torch.float32)
    w = np.random.default_rng(21).uniform(0.5, 1.5, D).astype(np.float32)
    cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
    ro, rfs = oracle.kda_recurrent(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["s0"], inp["cu"])
    ry = oracle.gate_norm(ro, inp["g"], w, 1e-6)
    for multi in (False, True):
        kw = {}
        if multi:
            lo, _ = kda.workspace_size(T, H, len(lens), max(lens))
            kw["workspace"] = torch.empty(lo, dtype=torch.uint8, device="cuda")
        y, fs = kda.chunk_fwd(q, k, v, la, b, s0, cu_seqlens=cu, max_seqlen=max(lens), gate=g,
                              norm_weight=dev(w, torch.float32), out_dtype=torch.float32, **kw)
        torch.cuda.synchronize()
        yh = host(y).reshape(T, H, D)
        check(yh, host(fs), ry, rfs)
        for n in range(len(lens)):
            sl = slice(inp["cu"][n], inp["cu"][n + 1])
            if lens[n]:
                assert_rel_l2(yh[sl], ry[sl], f"multi_pass={multi} seq {n} y")


@pytest.mark.parametrize("multi_pass", [False, True])
def test_prefill_state_checkpoints(multi_pass):
    """Prefix-cache checkpoints: checkpoint j of a sequence equals the oracle's
    final state after that sequence's first (j + 1) * 256 tokens; slots beyond a
    sequence's length stay untouched (zero)."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    lens, H, every = [700, 1100, 0, 513, 256], 2, 256
    inp = make_prefill(31, lens, H, bf16=True, init=True)
    T = inp["T"]
    dt = torch.bfloat16
    q, k, v, la = (dev(inp[x], dt).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha"))
    b = dev(inp["beta"], dt).view(1, T, H)
    cu = inp["cu"]
    kw = {}
    if multi_pass:
        lo, _ = kda.workspace_size(T, H, len(lens), max(lens))
        kw["workspace"] = torch.empty(lo, dtype=torch.uint8, device="cuda")
    ck_buf, ck_check = guarded_empty((len(lens), max(lens) // every, H, D, D), torch.float32)
    ck_buf.zero_()
    o, fs, ck = kda.chunk_fwd(q, k, v, la, b, dev(inp["s0"], torch.float32),
                              cu_seqlens=torch.from_numpy(cu.astype(np.int32)).cuda(), max_seqlen=max(lens),
                              checkpoints=ck_buf, ckpt_tokens=every, **kw)
    ck_check("checkpoints")
    ck = host(ck)
    assert ck.shape == (len(lens), max(lens) // every, H, D, D)
    for n, L in enumerate(lens):
        for j in range(ck.shape[1]):
            end = (j + 1) * every
            if end > L:
                assert not ck[n, j].any(), f"seq {n} checkpoint {j} written past the end"
                continue
            sl = slice(cu[n], cu[n] + end)
            _, ref = oracle.kda_recurrent(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["log_alpha"][sl],
                                          inp["beta"][sl], inp["s0"][n:n + 1])
            assert_rel_l2(ck[n, j], ref[0], f"seq {n} checkpoint {j}")
    # the last whole checkpoint of a sequence ending on a boundary is its final state
    np.testing.assert_array_equal(ck[4, 0], host(fs)[4])


@pytest.mark.parametrize("segments,gate,lens,memory", [
    (2, False, [256], "short"),
    (3, True, [300], "short"),
    (4, False, [700, 65, 0, 1, 200, 129], "short"),
    (8, True, [1000, 64, 450], "short"),
    (4, False, [700, 300], "long"),      # decays x 0.01: the state carries across segments
    (6, True, [900, 130], "none"),       # no decay at all: only the erase term forgets
])
def test_prefill_segment_parallel(segments, gate, lens, memory):
    """Segment-parallel prefill (segment maps, then segments from their folded
    initial states) against the oracle: outputs, final states, per sequence;
    sequences shorter than `segments` chunks leave empty segments.  The long- and
    no-decay cases make the segment maps matter (with the default decays the
    state forgets within a chunk)."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    H = 2
    kw = {"short": {}, "long": dict(la_scale=0.01), "none": dict(la_const=0.0)}[memory]
    inp = make_prefill(41 + segments, lens, H, bf16=True, gate=gate, init=True, **kw)
    T = inp["T"]
    dt = torch.bfloat16
    q, k, v, la = (dev(inp[x], dt).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha"))
    b = dev(inp["beta"], dt).view(1, T, H)
    g = dev(inp["g"], dt).view(1, T, H, D) if gate else None
    cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
    o, fs = kda.chunk_fwd(q, k, v, la, b, dev(inp["s0"], torch.float32), cu_seqlens=cu, max_seqlen=max(lens),
                          gate=g, out_dtype=torch.float32, segments=segments)
    torch.cuda.synchronize()
    ro, rfs = oracle_prefill(inp, gate=gate)
    oh, fh = host(o).reshape(T, H, D), host(fs)
    check(oh, fh, ro, rfs)
    for n, L in enumerate(lens):
        sl = slice(inp["cu"][n], inp["cu"][n + 1])
        if L:
            assert_rel_l2(oh[sl], ro[sl], f"seq {n}")
        assert_rel_l2(fh[n], rfs[n], f"seq {n} state")


# --------------------------------------- context parallelism across devices
# One process per device in production (linear_attention_recurrence_06_b200.kcp,
# exchange over NCCL); here the devices are emulated one after another on one
# GPU: every "rank" runs its transition, the stacked maps stand for the
# all-gather, then every rank composes its initial state and finishes.  No
# kernel waits on another.


def _kcp_pieces(L, R, ragged):
    """Cut points of a length-L sequence into R consecutive pieces."""
    if ragged:  # token boundaries off the chunk grid, one piece empty when R > 2
        cuts = [0] + [min(L, (L * (2 * r + 1)) // (2 * R) + 7 * r) for r in range(1, R)] + [L]
        if R > 2:
            cuts[2] = cuts[1]
    else:
        cuts = [(L * r) // R // 64 * 64 for r in range(R)] + [L]
    return [cuts[r + 1] - cuts[r] for r in range(R)]


@pytest.mark.parametrize("R,gate,lens,memory,ragged", [
    (2, False, [300], "short", False),
    (3, True, [700, 130], "long", True),
    (4, False, [1000, 64, 0, 257], "none", True),
    (8, True, [2048], "long", False),
])
def test_kcp_emulated_ranks(R, gate, lens, memory, ragged):
    """Each sequence cut into R consecutive pieces, piece r on rank r: per-rank
    transition, stacked maps, compose, finish.  The ranks' outputs, put back in
    order, and the last rank's final states equal the oracle over the whole
    sequences; a middle rank's state equals the oracle's state after its piece."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    H = 2
    kw = {"short": {}, "long": dict(la_scale=0.01), "none": dict(la_const=0.0)}[memory]
    inp = make_prefill(61 + R, lens, H, bf16=True, gate=gate, init=True, **kw)
    dt = torch.bfloat16
    pieces = [_kcp_pieces(L, R, ragged) for L in lens]
    ranks = []
    for r in range(R):
        idx, cu = [], [0]
        for n, L in enumerate(lens):
            a = int(inp["cu"][n]) + sum(pieces[n][:r])
            idx.extend(range(a, a + pieces[n][r]))
            cu.append(cu[-1] + pieces[n][r])
        idx = np.asarray(idx, dtype=np.int64)
        Tl = len(idx)
        loc = lambda x, last: dev(np.ascontiguousarray(inp[x][idx]), dt).view((1, Tl, H) + last)
        ranks.append(dict(idx=idx, T=Tl, cu=torch.tensor(cu, dtype=torch.int32, device="cuda"),
                          maxlen=max(int(np.diff(cu).max()), 0),
                          q=loc("q", (D,)), k=loc("k", (D,)), v=loc("v", (D,)), la=loc("log_alpha", (D,)),
                          b=loc("beta", ()), g=loc("g", (D,)) if gate else None))
    for rk in ranks:
        rk["trans"], rk["ws"] = kda.kcp_transition(rk["q"], rk["k"], rk["v"], rk["la"], rk["b"],
                                                   cu_seqlens=rk["cu"], max_seqlen=rk["maxlen"])
    gathered = torch.stack([rk["trans"] for rk in ranks])
    s0 = dev(inp["s0"], torch.float32)
    o_all = np.zeros((inp["T"], H, D))
    for r, rk in enumerate(ranks):
        s_in = kda.kcp_compose(gathered, r, s0)
        o, fs = kda.kcp_finish(s_in, rk["ws"], shape=(1, rk["T"], H, D), dtype=dt, cu_seqlens=rk["cu"],
                               max_seqlen=rk["maxlen"], gate=rk["g"], out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert kda.query_status(rk["ws"]) == 0
        o_all[rk["idx"]] = host(o).reshape(rk["T"], H, D)
        rk["fs"] = host(fs)
    ro, rfs = oracle_prefill(inp, gate=gate)
    check(o_all, ranks[-1]["fs"], ro, rfs)
    for n, L in enumerate(lens):
        sl = slice(inp["cu"][n], inp["cu"][n + 1])
        if L:
            assert_rel_l2(o_all[sl], ro[sl], f"seq {n}")
    # rank R//2's state: the oracle's state after pieces 0 .. R//2 of each sequence
    m = R // 2
    for n, L in enumerate(lens):
        end = int(inp["cu"][n]) + sum(pieces[n][:m + 1])
        sl = slice(int(inp["cu"][n]), end)
        _, ref = oracle.kda_recurrent(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["log_alpha"][sl],
                                      inp["beta"][sl], inp["s0"][n:n + 1])
        assert_rel_l2(ranks[m]["fs"][n], ref[0], f"seq {n} state after rank {m}")


def test_kcp_transition_is_the_oracle_segment_map():
    """(M, B) of kcp_transition against the oracle's segment transition, per
    head, on a ragged segment with long memory (M far from zero: the erase term
    shrinks it as the segment grows)."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    H, L = 2, 150
    inp = make_prefill(71, [L], H, bf16=True, la_scale=0.01)
    dt = torch.bfloat16
    q, k, v, la = (dev(inp[x], dt).view(1, L, H, D) for x in ("q", "k", "v", "log_alpha"))
    b = dev(inp["beta"], dt).view(1, L, H)
    trans, _ = kda.kcp_transition(q, k, v, la, b)
    torch.cuda.synchronize()
    t = host(trans)
    for h in range(H):
        M, B = oracle.segment_transition(inp["k"][:, h], inp["v"][:, h], inp["log_alpha"][:, h], inp["beta"][:, h])
        assert_rel_l2(t[0, 0, h], M, f"M head {h}")
        assert_rel_l2(t[1, 0, h], B, f"B head {h}")
        assert np.abs(M).max() > 0.1  # the segment map carries the state


def test_kcp_compose_is_the_fold():
    """kcp_compose against the fp64 fold S <- M_j S + B_j of the same fp32 maps."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    R, N, H = 5, 2, 3
    rng = np.random.default_rng(5)
    trans = rng.standard_normal((R, 2, N, H, D, D)).astype(np.float32)
    trans[:, 0] /= np.sqrt(D)  # spectral radius about 1
    s0 = rng.standard_normal((N, H, D, D)).astype(np.float32)
    g = torch.from_numpy(trans).cuda()
    for n_prev in (0, 1, 4):
        for init in (None, s0):
            out = host(kda.kcp_compose(g, n_prev, None if init is None else torch.from_numpy(init).cuda()))
            ref = np.zeros((N, H, D, D)) if init is None else init.astype(np.float64)
            for j in range(n_prev):
                ref = np.einsum("nhik,nhkc->nhic", trans[j, 0].astype(np.float64), ref) + trans[j, 1]
            assert rel_l2(out, ref) <= 1e-5 if n_prev else np.array_equal(out, ref)


def test_prefill_multi_pass_workspace():
    """A workspace that holds one chunk per sequence forces one pass per chunk:
    the state carried between passes must give the same result."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    lens = [200, 64, 1, 129]
    H = 2
    inp = make_prefill(9, lens, H, bf16=True, init=True)
    T = inp["T"]
    dt = torch.bfloat16
    q, k, v, la = (dev(inp[x], dt).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha"))
    b = dev(inp["beta"], dt).view(1, T, H)
    s0 = dev(inp["s0"], torch.float32)
    cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
    lo, _ = kda.workspace_size(T, H, len(lens), max(lens))
    ws = torch.empty(lo, dtype=torch.uint8, device="cuda")
    o, fs = kda.chunk_fwd(q, k, v, la, b, s0, cu_seqlens=cu, max_seqlen=max(lens), workspace=ws,
                          out_dtype=torch.float32)
    assert kda.query_status(ws) == 0
    ro, rfs = oracle_prefill(inp)
    check(host(o).reshape(T, H, D), host(fs), ro, rfs)


def test_prefill_in_place_state():
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    H = 2
    inp = make_prefill(13, [150], H, bf16=True, init=True)
    T = inp["T"]
    dt = torch.bfloat16
    q, k, v, la = (dev(inp[x], dt).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha"))
    b = dev(inp["beta"], dt).view(1, T, H)
    s = dev(inp["s0"], torch.float32)
    kda.chunk_fwd(q, k, v, la, b, s, final_state=s)
    torch.cuda.synchronize()
    _, rfs = oracle_prefill(inp)
    assert_rel_l2(host(s), rfs, "in-place final state")


# ------------------------------------------------------------------ decode


@pytest.mark.parametrize("scale", [1.0, 128 ** -0.5])
@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("gate", [False, True])
def test_decode_steps(bf16, gate, scale):
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    Bd, H, steps = 6, 3, 12
    dt = torch.bfloat16 if bf16 else torch.float32
    s_np = synth.states(0, Bd, H, D, D)
    s_dev = dev(s_np, torch.float32)
    s_ref = s_np.astype(np.float64)
    for step in range(steps):
        tb = synth.tokens(0, step * Bd, Bd, H, D, D, bf16=bf16, gate=gate)
        q, k, v, la = (dev(getattr(tb, x), dt) for x in ("q", "k", "v", "log_alpha"))
        b = dev(tb.beta, dt)
        g = dev(tb.g, dt) if gate else None
        o = kda.decode_step(s_dev, q, k, v, la, b, gate=g, out_dtype=torch.float32, scale=scale)
        ro, s_ref = oracle.decode_steps(s_ref, tb.q, tb.k, tb.v, tb.log_alpha, tb.beta, scale=scale)
        if gate:
            ro = oracle.gate_norm(ro, tb.g, None, 1e-6)
        torch.cuda.synchronize()
        assert_rel_l2(host(o), ro, f"step {step} o")
    assert_rel_l2(host(s_dev), s_ref, "state after the steps")


@pytest.mark.parametrize("bf16,gate,n,scale", [(True, False, 1, 1.0), (True, False, 4, 1.0), (True, True, 8, 1.0),
                                               (False, False, 3, 1.0), (True, False, 4, 128 ** -0.5),
                                               (False, True, 3, 0.125), (True, False, 17, 1.0),
                                               (False, False, 11, 128 ** -0.5)])
def test_decode_multi_step_with_step_states(bf16, gate, n, scale):
    """n consecutive steps in one call == n single steps of the oracle: every
    step's output, every step's state (for rollback) and the carried state.
    n = 11 and 17 cross the kernel's blocks of 8 staged token steps."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    Bd, H = 5, 3
    dt = torch.bfloat16 if bf16 else torch.float32
    s0 = synth.states(7, Bd, H, D, D)
    s_dev = dev(s0, torch.float32)
    toks = [synth.tokens(7, step * Bd, Bd, H, D, D, bf16=bf16, gate=gate) for step in range(n)]
    stack = lambda name: np.stack([getattr(tb, name) for tb in toks])
    q, k, v, la = (dev(stack(x), dt) for x in ("q", "k", "v", "log_alpha"))
    b = dev(stack("beta"), dt)
    g = dev(stack("g"), dt) if gate else None
    w = np.random.default_rng(7).uniform(0.5, 1.5, D).astype(np.float32) if gate else None
    o_buf, o_check = guarded_empty((n, Bd, H, D), torch.float32)
    st_buf, st_check = guarded_empty((n, Bd, H, D, D), torch.float32)
    o, states = kda.decode_steps(s_dev, q, k, v, la, b, gate=g, norm_weight=dev(w, torch.float32) if gate else None,
                                 out=o_buf, step_states=st_buf, scale=scale)
    o_check("o")
    st_check("step states")
    ref = s0.astype(np.float64)
    for step, tb in enumerate(toks):
        ro, ref = oracle.decode_steps(ref, tb.q, tb.k, tb.v, tb.log_alpha, tb.beta, scale=scale)
        if gate:
            ro = oracle.gate_norm(ro, tb.g, w, 1e-6)
        assert_rel_l2(host(o[step]), ro, f"step {step} output")
        assert_rel_l2(host(states[step]), ref, f"step {step} state")
    assert_rel_l2(host(s_dev), ref, "carried state")
    np.testing.assert_array_equal(host(s_dev), host(states[n - 1]))  # the carried state is the last step's


@pytest.mark.parametrize("n", [4, 10])
def test_decode_multi_step_matches_single_steps_exactly(n):
    """Carrying the state through n steps in registers gives the same bits as n
    separate one-step calls (same arithmetic, same order; n = 10 crosses a block
    of 8 staged token steps)."""
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    Bd, H = 4, 2
    s0 = synth.states(8, Bd, H, D, D)
    toks = [synth.tokens(8, step * Bd, Bd, H, D, D, bf16=True) for step in range(n)]
    stack = lambda name: dev(np.stack([getattr(tb, name) for tb in toks]), torch.bfloat16)
    q, k, v, la, b = (stack(x) for x in ("q", "k", "v", "log_alpha", "beta"))
    s_multi = dev(s0, torch.float32)
    o_multi = kda.decode_steps(s_multi, q, k, v, la, b, out_dtype=torch.float32)
    s_single = dev(s0, torch.float32)
    o_single = torch.stack([kda.decode_step(s_single, q[i], k[i], v[i], la[i], b[i], out_dtype=torch.float32)
                            for i in range(n)])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(o_multi), host(o_single))
    np.testing.assert_array_equal(host(s_multi), host(s_single))


# --------------------------------------------------------------- gate norm


@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("rows", [1000, 999, 1, 4097])
def test_gate_norm(bf16, rows):
    torch = _torch()
    import linear_attention_recurrence_06_b200 as kda
    dt = torch.bfloat16 if bf16 else torch.float32
    o = synth.normal(1, 100, (rows, D), 1.0, bf16)
    g = synth.normal(1, 101, (rows, D), 1.0, bf16)
    w = synth.normal(1, 102, (D,), 0.5, False) + 1.0
    y = kda.gate_norm(dev(o, dt), dev(g, dt), dev(w, torch.float32), out_dtype=torch.float32)
    ref = oracle.gate_norm(o.astype(np.float64), g, w, 1e-6)
    torch.cuda.synchronize()
    assert_rel_l2(host(y), ref, "y", tol=1e-5 if not bf16 else REL_L2_TOL)
