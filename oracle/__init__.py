"""fp64 CPU oracle for the KDA gated delta-rule recurrence (ctypes binding).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product path (the
CUDA library and its binding) never imports this package; the two share no
code.  The arithmetic lives in ``kda_oracle.c`` (plain loops, fp64); this file
only marshals numpy arrays.

Sources followed are cited in kda_oracle.c: the K3 article summaries on the
xhh.club tag page (items "KDA recurrence form", "chunkwise parallel
algorithm", "3:1 hybrid", "training and inference systems") and section 6 of
the nlpx.cn K3 paper walkthrough.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")

LOG_ALPHA_FLOOR = -5.0


def build(force: bool = False) -> str:
    """Compile the oracle shared library in place with gcc (-O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fvisibility=hidden",
               "-fno-fast-math", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _setup(lib):
    """Declares the argument types of the exported oracle functions."""
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    ci, cd = ctypes.c_int, ctypes.c_double
    lib.oracle_available_cores.restype = ci
    lib.oracle_kda_recurrent.argtypes = [f32p, f32p, f32p, f32p, f32p, f64p, i64p,
                                         ci, ci, ci, ci, ci, ci, cd, cd, ci, f64p, f64p, ci]
    lib.oracle_kda_recurrent.restype = ci
    lib.oracle_kda_chunkwise.argtypes = [f32p, f32p, f32p, f32p, f32p, f64p, i64p,
                                         ci, ci, ci, ci, ci, cd, cd, f64p, f64p, ci]
    lib.oracle_kda_chunkwise.restype = ci
    lib.oracle_kda_segment_transition.argtypes = [f32p, f32p, f32p, f32p, ci, ci, ci, cd,
                                                  f64p, f64p]
    lib.oracle_kda_segment_transition.restype = ci
    lib.oracle_kda_recurrent_bwd.argtypes = [f32p, f32p, f32p, f32p, f32p, f64p, i64p, f64p, f64p,
                                             ci, ci, ci, ci, cd, cd, f64p, f64p, f64p, f64p, f64p, f64p, ci]
    lib.oracle_kda_recurrent_bwd.restype = ci
    lib.oracle_gate_norm.argtypes = [f64p, f32p, f32p, cd, ctypes.c_int64, ci, f64p]
    lib.oracle_gate_norm.restype = ci
    return lib


def _L():
    global _lib
    if _lib is None:
        _lib = _setup(ctypes.CDLL(build()))
    return _lib


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def available_cores() -> int:
    return int(_L().oracle_available_cores())


def _cu(cu_seqlens, T):
    if cu_seqlens is None:
        return np.array([0, T], dtype=np.int64)
    return np.ascontiguousarray(cu_seqlens, dtype=np.int64)


def kda_recurrent(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, *,
                  scale: float = 1.0, la_floor: float = LOG_ALPHA_FLOOR, erase: bool = True,
                  heads=None, n_threads: int = 0, out=None, return_threads: bool = False):
    """Token-by-token recurrence (fp64).

    q, k, log_alpha: [T, H, dk]; v: [T, H, dv]; beta: [T, H] (packed tokens of
    N sequences delimited by cu_seqlens [N+1]; None = one sequence).
    init_state: [N, H, dk, dv] or None (zeros).  heads: (h_begin, h_end) to
    compute only those heads.  Returns (o [T,H,dv] fp64, final_state
    [N,H,dk,dv] fp64).
    """
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu = _cu(cu_seqlens, T)
    N = len(cu) - 1
    h0, h1 = heads if heads is not None else (0, H)
    q, qp = _f32(q); k, kp = _f32(k); v, vp = _f32(v)
    la, lp = _f32(log_alpha); b, bp = _f32(beta)
    if init_state is not None:
        s0, s0p = _f64(init_state)
    else:
        s0, s0p = None, ctypes.POINTER(ctypes.c_double)()
    o = out if out is not None else np.zeros((T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    nt = _L().oracle_kda_recurrent(qp, kp, vp, lp, bp, s0p, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                   N, H, dk, dv, h0, h1, scale, la_floor, int(erase),
                                   o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                   fs.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), n_threads)
    if nt < 0:
        raise ValueError("oracle_kda_recurrent: bad arguments")
    if return_threads:
        return o, fs, nt
    return o, fs


def kda_recurrent_bwd(q, k, v, log_alpha, beta, d_o, init_state=None, d_final=None, cu_seqlens=None, *,
                      scale: float = 1.0, la_floor: float = LOG_ALPHA_FLOOR, n_threads: int = 0):
    """Exact gradients of kda_recurrent (fp64, reverse sweep over the tokens).

    d_o: [T, H, dv] (dL/do); d_final: [N, H, dk, dv] or None (dL/d final state).
    Returns dict with dq, dk [T,H,dk], dv [T,H,dv], dbeta [T,H], dlog_alpha
    [T,H,dk] and d_init [N,H,dk,dv] (all fp64).  The clamp passes the gradient
    where log_alpha >= la_floor.
    """
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu = _cu(cu_seqlens, T)
    N = len(cu) - 1
    q, qp = _f32(q); k, kp = _f32(k); v, vp = _f32(v)
    la, lp = _f32(log_alpha); b, bp = _f32(beta)
    do, dop = _f64(d_o)
    P = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    null = ctypes.POINTER(ctypes.c_double)()
    if init_state is not None:
        s0, s0p = _f64(init_state)
    else:
        s0, s0p = None, null
    if d_final is not None:
        dfin, dfp = _f64(d_final)
    else:
        dfin, dfp = None, null
    out = dict(dq=np.zeros((T, H, dk)), dk=np.zeros((T, H, dk)), dv=np.zeros((T, H, dv)),
               dbeta=np.zeros((T, H)), dlog_alpha=np.zeros((T, H, dk)), d_init=np.zeros((N, H, dk, dv)))
    nt = _L().oracle_kda_recurrent_bwd(qp, kp, vp, lp, bp, s0p, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                       dop, dfp, N, H, dk, dv, scale, la_floor, P(out["dq"]), P(out["dk"]),
                                       P(out["dv"]), P(out["dbeta"]), P(out["dlog_alpha"]), P(out["d_init"]),
                                       n_threads)
    if nt < 0:
        raise ValueError("oracle_kda_recurrent_bwd: bad arguments")
    return out


def kda_chunkwise(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, *, chunk: int = 64,
                  scale: float = 1.0, la_floor: float = LOG_ALPHA_FLOOR, n_threads: int = 0):
    """Naive fp64 chunkwise form (matrix products inside chunks)."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu = _cu(cu_seqlens, T)
    N = len(cu) - 1
    q, qp = _f32(q); k, kp = _f32(k); v, vp = _f32(v)
    la, lp = _f32(log_alpha); b, bp = _f32(beta)
    if init_state is not None:
        s0, s0p = _f64(init_state)
    else:
        s0, s0p = None, ctypes.POINTER(ctypes.c_double)()
    o = np.zeros((T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _L().oracle_kda_chunkwise(qp, kp, vp, lp, bp, s0p, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                   N, H, dk, dv, chunk, scale, la_floor,
                                   o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                   fs.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), n_threads)
    if rc < 0:
        raise ValueError("oracle_kda_chunkwise: bad arguments")
    return o, fs


def segment_transition(k, v, log_alpha, beta, *, la_floor: float = LOG_ALPHA_FLOOR):
    """(M [dk,dk], B [dk,dv]) with S_out = M S_in + B over one head's segment.

    k, log_alpha: [L, dk]; v: [L, dv]; beta: [L].
    """
    L, dk = k.shape
    dv = v.shape[-1]
    k, kp = _f32(k); v, vp = _f32(v); la, lp = _f32(log_alpha); b, bp = _f32(beta)
    M = np.zeros((dk, dk), dtype=np.float64)
    B = np.zeros((dk, dv), dtype=np.float64)
    rc = _L().oracle_kda_segment_transition(kp, vp, lp, bp, L, dk, dv, la_floor,
                                            M.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                            B.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc < 0:
        raise ValueError("oracle_kda_segment_transition: bad arguments")
    return M, B


def gate_norm(o, g, w=None, eps: float = 1e-6):
    """Per-head RMSNorm over dv, times w, times sigmoid(g) (fp64)."""
    o, op = _f64(o)
    g, gp = _f32(g)
    dv = o.shape[-1]
    rows = o.size // dv
    if w is not None:
        w, wp = _f32(w)
    else:
        wp = ctypes.POINTER(ctypes.c_float)()
    y = np.zeros(o.shape, dtype=np.float64)
    rc = _L().oracle_gate_norm(op, gp, wp, eps, rows, dv, y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc < 0:
        raise ValueError("oracle_gate_norm: bad arguments")
    return y


def decode_steps(state, q, k, v, log_alpha, beta, *, scale: float = 1.0, n_threads: int = 0):
    """One recurrent step for each of Bd independent sequences.

    state: [Bd, H, dk, dv] (fp64 or fp32); q, k, log_alpha: [Bd, H, dk];
    v: [Bd, H, dv]; beta: [Bd, H].  Returns (o [Bd,H,dv], new_state).
    A decode step is the recurrence run for one token per sequence.
    """
    Bd = q.shape[0]
    cu = np.arange(Bd + 1, dtype=np.int64)
    return kda_recurrent(q, k, v, log_alpha, beta, init_state=state, cu_seqlens=cu,
                         scale=scale, n_threads=n_threads)
