"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

None of these compares the oracle with a re-typed copy of itself: each check is
a hand-worked example, a closed form, an invariant, a reduction to a textbook
special case (linear attention, DeltaNet associative memory), brute force on
tiny inputs, or an independent formulation (naive chunkwise, segment maps).
Sources: the K3 article summaries on the xhh.club tag page (items "KDA
recurrence form", "chunkwise parallel algorithm", "training and inference
systems") and section 6 (terminology / self-test) of the nlpx.cn K3 paper
walkthrough.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_steps.json")
rng_global = np.random.default_rng(1234)


def rand_inputs(T, H, dk, dv, rng, unit_k=True, la_lo=-5.0, beta=None):
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    k = k.astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    la = rng.uniform(la_lo, 0.0, (T, H, dk)).astype(np.float32)
    b = (rng.uniform(0, 1, (T, H)) if beta is None else np.full((T, H), beta)).astype(np.float32)
    return q, k, v, la, b


def exact_unit_keys(T, H, dk, rng):
    """Keys with entries +-1/sqrt(dk), dk a power of 4: unit norm exactly in float32."""
    assert dk in (1, 4, 16, 64)
    s = rng.choice([-1.0, 1.0], size=(T, H, dk)) / np.sqrt(dk)
    return s.astype(np.float32)


# ---------------------------------------------------------------- hand-worked


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    dk, dv = case["dk"], case["dv"]
    T = len(case["beta"])
    q = np.array(case["q"], np.float32).reshape(T, 1, dk)
    k = np.array(case["k"], np.float32).reshape(T, 1, dk)
    v = np.array(case["v"], np.float32).reshape(T, 1, dv)
    la = np.array(case["log_alpha"], np.float32).reshape(T, 1, dk)
    b = np.array(case["beta"], np.float32).reshape(T, 1)
    s0 = np.array(case["S0"], np.float64).reshape(1, 1, dk, dv)
    o, fs = oracle.kda_recurrent(q, k, v, la, b, s0)
    # tolerance: float32 rounding of the inputs (0.6, 0.8, ln 0.5)
    np.testing.assert_allclose(o[:, 0, :], np.array(case["o"]), rtol=0, atol=2e-6)
    np.testing.assert_allclose(fs[0, 0], np.array(case["S_T"]), rtol=0, atol=2e-6)


# ------------------------------------------------------- erase-write (I1)


@pytest.mark.parametrize("dk", [4, 16, 64])
def test_erase_write_invariant(dk):
    """beta=1 and |k|=1: right after step t the state returns exactly v_t for k_t,
    whatever the decay and the previous state (erase-then-write)."""
    rng = np.random.default_rng(dk)
    T, H, dv = 40, 2, 8
    q, _, v, la, _ = rand_inputs(T, H, dk, dv, rng)
    k = exact_unit_keys(T, H, dk, rng)
    b = np.ones((T, H), np.float32)
    s = rng.standard_normal((1, H, dk, dv))
    for t in range(T):
        _, s = oracle.kda_recurrent(q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1], b[t:t + 1], s)
        recalled = np.einsum("hij,hi->hj", s[0], k[t].astype(np.float64))
        np.testing.assert_allclose(recalled, v[t], rtol=0, atol=1e-12)


# ------------------------------------- DeltaNet associative memory (I2)


def test_deltanet_orthonormal_keys_store_all_pairs():
    """No decay, beta=1, orthonormal keys: after writing (k_i, v_i) for all i the
    state returns every v_i for its k_i and leaves the orthogonal complement of
    the keys exactly as S0 had it (DeltaNet as an associative memory)."""
    rng = np.random.default_rng(7)
    dk, dv, T = 16, 5, 10
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :T].T.copy()               # T orthonormal rows
    k = keys.reshape(T, 1, dk).astype(np.float32)
    keys32 = k[:, 0, :].astype(np.float64)
    v = rng.standard_normal((T, 1, dv)).astype(np.float32)
    q = np.zeros((T, 1, dk), np.float32)
    la = np.zeros((T, 1, dk), np.float32)
    b = np.ones((T, 1), np.float32)
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, fs = oracle.kda_recurrent(q, k, v, la, b, s0)
    S = fs[0, 0]
    # float32 keys are orthonormal only to ~1e-7
    np.testing.assert_allclose(keys32 @ S, v[:, 0, :], atol=5e-6)
    perp = Qm[:, T:].T
    np.testing.assert_allclose(perp @ S, perp @ s0[0, 0], atol=5e-6)


@pytest.mark.parametrize("beta", [0.25, 0.5, 0.9])
def test_repeated_key_geometric_convergence(beta):
    """Same unit key, same value, no decay, empty start: after n writes the
    state returns v (1 - (1-beta)^n) for that key."""
    dk, dv, n = 16, 3, 12
    rng = np.random.default_rng(3)
    kk = exact_unit_keys(1, 1, dk, rng)[0, 0]
    k = np.tile(kk, (n, 1, 1)).reshape(n, 1, dk)
    v1 = rng.standard_normal(dv).astype(np.float32)
    v = np.tile(v1, (n, 1, 1)).reshape(n, 1, dv)
    q = np.tile(kk, (n, 1, 1)).reshape(n, 1, dk)      # read with the key itself
    la = np.zeros((n, 1, dk), np.float32)
    b = np.full((n, 1), beta, np.float32)
    o, _ = oracle.kda_recurrent(q, k, v, la, b)
    beta64 = float(np.float32(beta))
    for t in range(n):
        np.testing.assert_allclose(o[t, 0], v1.astype(np.float64) * (1 - (1 - beta64) ** (t + 1)), rtol=1e-12, atol=1e-12)


# ---------------------------------------------- linear attention lineage (I3)


def test_linear_attention_reduction_bruteforce():
    """Erase dropped, write coefficient 1, no decay: causal linear attention,
    o_t = S0^T q_t + sum_{s<=t} (k_s . q_t) v_s (O(T^2) brute force)."""
    rng = np.random.default_rng(11)
    T, H, dk, dv = 37, 3, 8, 6
    q, k, v, _, _ = rand_inputs(T, H, dk, dv, rng, unit_k=False)
    la = np.zeros((T, H, dk), np.float32)
    b = np.ones((T, H), np.float32)
    s0 = rng.standard_normal((1, H, dk, dv))
    o, _ = oracle.kda_recurrent(q, k, v, la, b, s0, erase=False)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    ref = np.zeros((T, H, dv))
    for t in range(T):
        for h in range(H):
            acc = s0[0, h].T @ q64[t, h]
            for s in range(t + 1):
                acc = acc + (k64[s, h] @ q64[t, h]) * v64[s, h]
            ref[t, h] = acc
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_gated_linear_attention_closed_form():
    """Erase dropped, per-channel decay on: gated linear attention in closed form
    with the global cumulative log-decay G (G_t includes step t):
    o_t = sum_c q_tc e^{G_tc} S0[c,:] + sum_{s<=t} beta_s sum_c q_tc k_sc e^{G_tc-G_sc} v_s.
    Pins which step's decay applies to which write (per key channel)."""
    rng = np.random.default_rng(12)
    T, H, dk, dv = 29, 2, 8, 4
    q, k, v, la, b = rand_inputs(T, H, dk, dv, rng, unit_k=False, la_lo=-1.0)
    s0 = rng.standard_normal((1, H, dk, dv))
    o, fs = oracle.kda_recurrent(q, k, v, la, b, s0, erase=False)
    q64, k64, v64, b64 = (x.astype(np.float64) for x in (q, k, v, b))
    G = np.cumsum(la.astype(np.float64), axis=0)
    ref = np.zeros((T, H, dv))
    for t in range(T):
        for h in range(H):
            acc = (q64[t, h] * np.exp(G[t, h])) @ s0[0, h]
            for s in range(t + 1):
                w = np.sum(q64[t, h] * k64[s, h] * np.exp(G[t, h] - G[s, h]))
                acc = acc + b64[s, h] * w * v64[s, h]
            ref[t, h] = acc
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-11)
    Sref = np.exp(G[-1])[:, :, None] * s0[0] + sum(
        b64[s][:, None, None] * (k64[s] * np.exp(G[-1] - G[s]))[:, :, None] * v64[s][:, None, :]
        for s in range(T))
    np.testing.assert_allclose(fs[0], Sref, rtol=1e-11, atol=1e-11)


# --------------------------------------------------------- beta = 0 (I4)


def test_beta_zero_pure_decay():
    """beta = 0: nothing is written or erased; the state only decays per key
    channel (rows): S_t = Diag(exp(sum_{r<=t} l_r)) S0, o_t = S_t^T q_t."""
    rng = np.random.default_rng(5)
    T, H, dk, dv = 21, 2, 6, 9
    q, k, v, la, _ = rand_inputs(T, H, dk, dv, rng)
    b = np.zeros((T, H), np.float32)
    s0 = rng.standard_normal((1, H, dk, dv))
    o, fs = oracle.kda_recurrent(q, k, v, la, b, s0)
    G = np.cumsum(la.astype(np.float64), axis=0)
    for t in range(T):
        St = np.exp(G[t])[:, :, None] * s0[0]
        np.testing.assert_allclose(o[t], np.einsum("hij,hi->hj", St, q[t].astype(np.float64)),
                                   rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fs[0], np.exp(G[-1])[:, :, None] * s0[0], rtol=1e-12, atol=1e-14)


def test_log_decay_floor():
    """log-decay values below -5 act as -5 (the bound the pages fix)."""
    rng = np.random.default_rng(6)
    T, H, dk, dv = 9, 1, 4, 4
    q, k, v, la, b = rand_inputs(T, H, dk, dv, rng)
    la_low = la.copy()
    la_low[::2] = -12.0
    la_clamped = la.copy()
    la_clamped[::2] = -5.0
    o1, f1 = oracle.kda_recurrent(q, k, v, la_low, b)
    o2, f2 = oracle.kda_recurrent(q, k, v, la_clamped, b)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(f1, f2)
    # and the bound is really in effect: without it the results differ
    o3, _ = oracle.kda_recurrent(q, k, v, la_low, b, la_floor=-100.0)
    assert np.max(np.abs(o3 - o1)) > 1e-6


def test_output_scale_is_linear():
    rng = np.random.default_rng(8)
    q, k, v, la, b = rand_inputs(17, 2, 8, 8, rng)
    o1, f1 = oracle.kda_recurrent(q, k, v, la, b, scale=1.0)
    o2, f2 = oracle.kda_recurrent(q, k, v, la, b, scale=0.125)
    np.testing.assert_allclose(o2, 0.125 * o1, rtol=1e-15)
    np.testing.assert_array_equal(f1, f2)


# ------------------------------------------- chunkwise == recurrence (I5)


@pytest.mark.parametrize("C", [1, 2, 16, 64])
@pytest.mark.parametrize("lengths", [[1], [5], [63], [64], [65], [200], [3, 64, 130, 17]])
def test_chunkwise_equals_recurrence(C, lengths):
    """The chunkwise form (matrix products inside chunks, recurrence between
    them) reaches the same result as the token recurrence."""
    rng = np.random.default_rng(C * 1000 + sum(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T, H, dk, dv = int(cu[-1]), 2, 16, 12
    q, k, v, la, b = rand_inputs(T, H, dk, dv, rng)
    s0 = 0.1 * rng.standard_normal((len(lengths), H, dk, dv))
    o1, f1 = oracle.kda_recurrent(q, k, v, la, b, s0, cu)
    o2, f2 = oracle.kda_chunkwise(q, k, v, la, b, s0, cu, chunk=C)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-10 * max(1.0, np.abs(o1).max()))
    np.testing.assert_allclose(f2, f1, rtol=0, atol=1e-10 * max(1.0, np.abs(f1).max()))


def test_chunkwise_equals_recurrence_full_width_steep_decay():
    """dk = dv = 128 with every log-decay at the -5 floor (largest exponent
    spans inside a 64-token chunk)."""
    rng = np.random.default_rng(99)
    T, H, dk, dv = 150, 1, 128, 128
    q, k, v, _, b = rand_inputs(T, H, dk, dv, rng)
    la = np.full((T, H, dk), -5.0, np.float32)
    o1, f1 = oracle.kda_recurrent(q, k, v, la, b)
    o2, f2 = oracle.kda_chunkwise(q, k, v, la, b, chunk=64)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-10 * np.abs(o1).max())


# ----------------------------------------- segment transitions (I6)


def test_segment_transition_is_the_state_map():
    """S_out = M S_in + B for any S_in over a segment (affine state map)."""
    rng = np.random.default_rng(21)
    L, dk, dv = 23, 8, 5
    q, k, v, la, b = rand_inputs(L, 1, dk, dv, rng)
    M, B = oracle.segment_transition(k[:, 0], v[:, 0], la[:, 0], b[:, 0])
    for _ in range(3):
        s_in = rng.standard_normal((1, 1, dk, dv))
        _, s_out = oracle.kda_recurrent(q, k, v, la, b, s_in)
        np.testing.assert_allclose(s_out[0, 0], M @ s_in[0, 0] + B, rtol=0, atol=1e-12)


def test_segment_composition_associative_not_additive():
    """Composing segment maps (M2 M1, M2 B1 + B2) equals running the segments
    in sequence (associative prefix scan); summing per-segment states does not."""
    rng = np.random.default_rng(22)
    lens = [17, 9, 30]
    dk, dv = 8, 6
    T = sum(lens)
    q, k, v, la, b = rand_inputs(T, 1, dk, dv, rng)
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, full = oracle.kda_recurrent(q, k, v, la, b, s0)
    maps, t0 = [], 0
    for L in lens:
        sl = slice(t0, t0 + L)
        maps.append(oracle.segment_transition(k[sl, 0], v[sl, 0], la[sl, 0], b[sl, 0]))
        t0 += L
    # left fold and a different bracketing give the same map
    def comp(a, bmap):  # apply a then bmap
        return bmap[0] @ a[0], bmap[0] @ a[1] + bmap[1]
    m12_3 = comp(comp(maps[0], maps[1]), maps[2])
    m1_23 = comp(maps[0], comp(maps[1], maps[2]))
    for Mx, Bx in (m12_3, m1_23):
        np.testing.assert_allclose(Mx @ s0[0, 0] + Bx, full[0, 0], rtol=0, atol=1e-11)
    # plain summation of independently-run segment states is wrong
    summed = np.zeros((dk, dv))
    t0 = 0
    for i, L in enumerate(lens):
        sl = slice(t0, t0 + L)
        _, fs_i = oracle.kda_recurrent(q[sl], k[sl], v[sl], la[sl], b[sl], s0 if i == 0 else None)
        summed += fs_i[0, 0]
        t0 += L
    assert np.abs(summed - full[0, 0]).max() > 1e-3


# -------------------------------------------- dv separability (I7)


def test_value_columns_are_independent():
    rng = np.random.default_rng(31)
    T, H, dk, dv = 40, 2, 8, 12
    q, k, v, la, b = rand_inputs(T, H, dk, dv, rng)
    s0 = rng.standard_normal((1, H, dk, dv))
    o, fs = oracle.kda_recurrent(q, k, v, la, b, s0)
    cols = [1, 4, 5, 11]
    o2, fs2 = oracle.kda_recurrent(q, k, v[:, :, cols], la, b, s0[:, :, :, cols])
    np.testing.assert_allclose(o2, o[:, :, cols], rtol=0, atol=1e-13)
    np.testing.assert_allclose(fs2, fs[:, :, :, cols], rtol=0, atol=1e-13)


# --------------------------------------------------- contraction (I8)


def test_transition_is_a_contraction():
    """|k| = 1, beta in [0,1], decays <= 1: ||S_t - beta k v^T||_F <= ||S_{t-1}||_F."""
    rng = np.random.default_rng(41)
    T, H, dk, dv = 60, 1, 16, 16
    q, _, v, la, b = rand_inputs(T, H, dk, dv, rng, la_lo=-0.3)
    k = exact_unit_keys(T, H, dk, rng)
    s = 3.0 * rng.standard_normal((1, H, dk, dv))
    for t in range(T):
        prev = np.linalg.norm(s[0, 0])
        _, s = oracle.kda_recurrent(q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1], b[t:t + 1], s)
        write = float(b[t, 0]) * np.outer(k[t, 0].astype(np.float64), v[t, 0].astype(np.float64))
        assert np.linalg.norm(s[0, 0] - write) <= prev * (1 + 1e-12)


# ------------------------------------------------------ gate + norm (I9)


def test_gate_norm_closed_forms():
    rng = np.random.default_rng(51)
    rows, dv, eps = 33, 128, 1e-6
    o = rng.standard_normal((rows, dv))
    # gate fully open, unit weight: RMS(y) = 1/sqrt(1 + eps/ms)
    y = oracle.gate_norm(o, np.full((rows, dv), 40.0, np.float32), None, eps)
    ms = np.mean(o * o, axis=1)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=1)), 1 / np.sqrt(1 + eps / ms), rtol=1e-12)
    # gate at zero halves it; direction is preserved
    y0 = oracle.gate_norm(o, np.zeros((rows, dv), np.float32), None, eps)
    np.testing.assert_allclose(y0 * 2 * np.sqrt(ms + eps)[:, None], o, rtol=1e-12)
    # zero rows stay zero
    yz = oracle.gate_norm(np.zeros((4, dv)), rng.standard_normal((4, dv)).astype(np.float32), None, eps)
    assert np.all(yz == 0)
    # per-channel weight multiplies channel-wise
    w = rng.uniform(0.5, 2, dv).astype(np.float32)
    g = rng.standard_normal((rows, dv)).astype(np.float32)
    np.testing.assert_allclose(oracle.gate_norm(o, g, w, eps), oracle.gate_norm(o, g, None, eps) * w,
                               rtol=1e-12)
    # scale invariance of the norm (eps aside)
    np.testing.assert_allclose(oracle.gate_norm(1000 * o, g, None, 0.0), oracle.gate_norm(o, g, None, 0.0),
                               rtol=1e-12)


# ------------------------------------------------------ composition (I10)


def test_varlen_packed_equals_separate_runs():
    rng = np.random.default_rng(61)
    lens = [5, 64, 1, 70, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T, H, dk, dv = int(cu[-1]), 2, 8, 8
    q, k, v, la, b = rand_inputs(T, H, dk, dv, rng)
    s0 = rng.standard_normal((len(lens), H, dk, dv))
    o, fs = oracle.kda_recurrent(q, k, v, la, b, s0, cu)
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        on, fn = oracle.kda_recurrent(q[sl], k[sl], v[sl], la[sl], b[sl], s0[n:n + 1])
        np.testing.assert_array_equal(on, o[sl])
        np.testing.assert_array_equal(fn[0], fs[n])


def test_prefill_then_decode_equals_one_pass():
    rng = np.random.default_rng(71)
    T, n_dec, H, dk, dv = 50, 7, 2, 8, 8
    q, k, v, la, b = rand_inputs(T + n_dec, H, dk, dv, rng)
    o_all, f_all = oracle.kda_recurrent(q, k, v, la, b)
    _, s = oracle.kda_recurrent(q[:T], k[:T], v[:T], la[:T], b[:T])
    for t in range(T, T + n_dec):
        o_t, s = oracle.decode_steps(s, q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1], b[t:t + 1])
        np.testing.assert_allclose(o_t[0], o_all[t], rtol=0, atol=1e-13)
    np.testing.assert_allclose(s, f_all, rtol=0, atol=1e-13)


def test_heads_subset_matches_full():
    rng = np.random.default_rng(81)
    q, k, v, la, b = rand_inputs(20, 4, 8, 8, rng)
    o, fs = oracle.kda_recurrent(q, k, v, la, b)
    o2, fs2 = oracle.kda_recurrent(q, k, v, la, b, heads=(1, 3))
    np.testing.assert_array_equal(o2[:, 1:3], o[:, 1:3])
    np.testing.assert_array_equal(fs2[:, 1:3], fs[:, 1:3])
    assert np.all(o2[:, 0] == 0) and np.all(o2[:, 3] == 0)


# ------------------------------------------- backward (exact gradients, I11)
# The pages give no backward; the oracle's is the exact gradient of its forward.
# Pinned by central finite differences of the fp64 forward: a scalar loss
#   L = sum(d_o * o) + sum(d_final * S_final)
# is perturbed in every element of every input; the difference quotient uses
# the perturbation actually representable in float32.

BWD_LENS = [5, 4]
BWD_SCALE = 0.7


def _bwd_case(seed=31, la_lo=-1.5):
    rng = np.random.default_rng(seed)
    T, H, dk, dv = sum(BWD_LENS), 2, 4, 3
    q, k, v, la, b = rand_inputs(T, H, dk, dv, rng, unit_k=False, la_lo=la_lo)
    s0 = rng.standard_normal((len(BWD_LENS), H, dk, dv))
    d_o = rng.standard_normal((T, H, dv))
    d_fin = rng.standard_normal((len(BWD_LENS), H, dk, dv))
    cu = np.cumsum([0] + BWD_LENS)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b), s0, d_o, d_fin, cu


def _loss(x, s0, d_o, d_fin, cu):
    o, fs = oracle.kda_recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], s0, cu, scale=BWD_SCALE,
                                 n_threads=1)
    return float((o * d_o).sum() + (fs * d_fin).sum())


def _fd(x, name, idx, s0, d_o, d_fin, cu, h=1e-3):
    base = x[name][idx]
    hi, lo = np.float32(base + h), np.float32(base - h)
    xp = {kk: vv.copy() for kk, vv in x.items()}
    xp[name][idx] = hi
    lp = _loss(xp, s0, d_o, d_fin, cu)
    xp[name][idx] = lo
    lm = _loss(xp, s0, d_o, d_fin, cu)
    return (lp - lm) / (float(hi) - float(lo))


def test_backward_matches_finite_differences():
    x, s0, d_o, d_fin, cu = _bwd_case()
    g = oracle.kda_recurrent_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o, s0, d_fin, cu,
                                 scale=BWD_SCALE, n_threads=1)
    names = dict(q="dq", k="dk", v="dv", log_alpha="dlog_alpha", beta="dbeta")
    for name, gname in names.items():
        for idx in np.ndindex(*x[name].shape):
            fd = _fd(x, name, idx, s0, d_o, d_fin, cu)
            an = g[gname][idx]
            assert abs(fd - an) <= 2e-5 * max(1.0, abs(an)), f"{gname}{idx}: fd {fd} analytic {an}"
    # initial state (fp64 input): plain central differences
    for idx in np.ndindex(*s0.shape):
        sp, sm = s0.copy(), s0.copy()
        sp[idx] += 1e-4
        sm[idx] -= 1e-4
        fd = (_loss(x, sp, d_o, d_fin, cu) - _loss(x, sm, d_o, d_fin, cu)) / 2e-4
        assert abs(fd - g["d_init"][idx]) <= 1e-6 * max(1.0, abs(fd)), f"d_init{idx}"


def test_backward_clamp_blocks_gradient():
    """Log-decays below the floor get no gradient (the clamp is flat there);
    above it the gradient matches finite differences."""
    x, s0, d_o, d_fin, cu = _bwd_case(seed=32, la_lo=-8.0)
    g = oracle.kda_recurrent_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_o, s0, d_fin, cu,
                                 scale=BWD_SCALE, n_threads=1)
    below = x["log_alpha"] < -5.0 - 1e-3
    above = x["log_alpha"] > -5.0 + 1e-3
    assert below.any() and above.any()
    assert np.all(g["dlog_alpha"][below] == 0.0)
    for idx in zip(*np.nonzero(above)):
        fd = _fd(x, "log_alpha", idx, s0, d_o, d_fin, cu)
        assert abs(fd - g["dlog_alpha"][idx]) <= 2e-5 * max(1.0, abs(fd))
    assert np.abs(g["dlog_alpha"][above]).max() > 1e-4  # the comparison is not vacuous


def test_backward_of_one_token_closed_form():
    """One token from a zero state: o = scale (q.k) beta v, so dv = scale beta (q.k) d_o,
    dbeta = scale (q.k) (v.d_o), dq = scale beta (v.d_o) k; the decay does not act
    (zero state), so dlog_alpha = 0."""
    rng = np.random.default_rng(33)
    q, k, v, la, b = rand_inputs(1, 1, 5, 3, rng, unit_k=False)
    d_o = rng.standard_normal((1, 1, 3))
    g = oracle.kda_recurrent_bwd(q, k, v, la, b, d_o, scale=0.5, n_threads=1)
    qk = float(np.dot(q[0, 0].astype(np.float64), k[0, 0]))
    vd = float(np.dot(v[0, 0].astype(np.float64), d_o[0, 0]))
    bb = float(b[0, 0])
    np.testing.assert_allclose(g["dv"][0, 0], 0.5 * bb * qk * d_o[0, 0], rtol=1e-12)
    np.testing.assert_allclose(g["dbeta"][0, 0], 0.5 * qk * vd, rtol=1e-12)
    np.testing.assert_allclose(g["dq"][0, 0], 0.5 * bb * vd * k[0, 0].astype(np.float64), rtol=1e-12)
    np.testing.assert_allclose(g["dk"][0, 0], 0.5 * bb * vd * q[0, 0].astype(np.float64), rtol=1e-12)
    assert np.all(g["dlog_alpha"] == 0.0)
