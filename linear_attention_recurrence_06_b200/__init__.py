"""KDA (Kimi Delta Attention) gated delta-rule recurrence on B200 (sm_100a).

Thin Python binding of ``libkda.so`` (C ABI in ``include/kda.h``).  This module
only marshals arguments: it checks shapes, allocates outputs and the workspace
with torch (device memory and streams are all torch is used for) and calls the
library.  Every step of the computation runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback.  If the library is missing or no CUDA
device is present the calls raise.

Entry points (same names as the C ABI):
  chunk_fwd      chunkwise prefill: (o or y, final_state)
  decode_step    one recurrent step per sequence, state updated in place
  gate_norm      per-head RMSNorm over dv times sigmoid output gate
  workspace_size bytes the prefill needs
  chunk_bwd      gradients of the prefill (without the gate)
  kcp_transition / kcp_compose / kcp_finish
                 the per-device steps of context parallelism across devices
                 (the exchange between them is in ``kcp.py``)
  query_status   reads and clears the device status word of a workspace
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK = 0
KDA_F32, KDA_BF16 = 0, 1
HEAD_DIM = 128

_STATUS_NAMES = {
    0: "KDA_OK", -1: "KDA_ERR_INVALID_ARG", -2: "KDA_ERR_UNSUPPORTED", -3: "KDA_ERR_MISALIGNED",
    -4: "KDA_ERR_WORKSPACE", -5: "KDA_ERR_CUDA", -6: "KDA_ERR_TIMEOUT", -7: "KDA_ERR_DEVICE_ARG",
}


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 16), ("launches", ctypes.c_int), ("ms", ctypes.c_double)]


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS_NAMES.get(status, status)} ({status})")


_lib = None


def load_library(path: str | None = None):
    """Loads libkda.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with `python -m linear_attention_recurrence_06_b200.build` "
                          "(there is no fallback implementation)")
    lib = ctypes.CDLL(p)
    vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [i32]
    lib.kda_version.restype = i32
    lib.kda_chunk_fwd_workspace_size.restype = i32
    lib.kda_chunk_fwd_workspace_size.argtypes = [i64, i32, i32, i32, i32, i64, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.kda_chunk_fwd.restype = i32
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, vp, i32, i64,
                                  i32, i32, f32, vp, vp, f32, vp, sz, vp]
    lib.kda_chunk_fwd_ckpt.restype = i32
    lib.kda_chunk_fwd_ckpt.argtypes = list(lib.kda_chunk_fwd.argtypes[:22]) + [vp, i64] + \
        list(lib.kda_chunk_fwd.argtypes[22:])
    lib.kda_chunk_fwd_segmented.restype = i32
    lib.kda_chunk_fwd_segmented.argtypes = list(lib.kda_chunk_fwd.argtypes[:22]) + [i32] + \
        list(lib.kda_chunk_fwd.argtypes[22:])
    lib.kda_chunk_fwd_segmented_workspace_size.restype = i32
    lib.kda_chunk_fwd_segmented_workspace_size.argtypes = [i64, i32, i32, i32, i32, i64, i32, ctypes.POINTER(sz)]
    lib.kda_kcp_workspace_size.restype = i32
    lib.kda_kcp_workspace_size.argtypes = [i64, i32, i32, i32, i32, i64, ctypes.POINTER(sz)]
    lib.kda_kcp_transition.restype = i32
    lib.kda_kcp_transition.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, vp, i32, i64, i32, f32, vp, vp,
                                       sz, vp]
    lib.kda_kcp_compose.restype = i32
    lib.kda_kcp_compose.argtypes = [vp, i32, vp, vp, i32, i32, i32, i32, vp]
    lib.kda_kcp_finish.restype = i32
    lib.kda_kcp_finish.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, vp, i32, i64, i32, i32, vp, vp, f32, vp, sz,
                                   vp]
    lib.kda_chunk_bwd_workspace_size.restype = i32
    lib.kda_chunk_bwd_workspace_size.argtypes = [i64, i32, i32, i32, i32, i64, ctypes.POINTER(sz)]
    lib.kda_chunk_bwd.restype = i32
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                  vp, i32, i64, i32, f32, vp, sz, vp]
    lib.kda_decode_step.restype = i32
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, f32, vp]
    lib.kda_decode_steps.restype = i32
    lib.kda_decode_steps.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, vp, vp, f32,
                                     vp, vp]
    lib.kda_gate_norm.restype = i32
    lib.kda_gate_norm.argtypes = [vp, vp, vp, f32, vp, i64, i32, i32, i32, vp]
    lib.kda_query_status.restype = i32
    lib.kda_query_status.argtypes = [vp, vp]
    lib.kda_chunk_fwd_noalloc.restype = i32
    lib.kda_chunk_fwd_noalloc.argtypes = list(lib.kda_chunk_fwd.argtypes[:22]) + [vp]
    lib.kda_chunk_fwd_noalloc_query_status.restype = i32
    lib.kda_chunk_fwd_noalloc_query_status.argtypes = [vp]
    lib.kda_test_drop_tile_load.restype = i32
    lib.kda_test_drop_tile_load.argtypes = [ctypes.c_ulonglong]
    lib.kda_profile_enable.restype = i32
    lib.kda_profile_enable.argtypes = [i32]
    lib.kda_profile_read.restype = i32
    lib.kda_profile_read.argtypes = [ctypes.POINTER(KernelTime), i32, ctypes.POINTER(i32)]
    if path is None:
        _lib = lib
    return lib


def _torch():
    import torch
    return torch


def _dt(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("all tensors must be CUDA tensors (there is no CPU path)")
            if not t.is_contiguous():
                raise ValueError("all tensors must be contiguous")


def segmented_workspace_size(T: int, H: int, n_seqs: int, max_seqlen: int, segments: int, dk: int = HEAD_DIM,
                             dv: int = HEAD_DIM) -> int:
    """Workspace bytes of the segment-parallel prefill."""
    n = ctypes.c_size_t(0)
    st = load_library().kda_chunk_fwd_segmented_workspace_size(T, H, dk, dv, n_seqs, max_seqlen, segments,
                                                               ctypes.byref(n))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_segmented_workspace_size")
    return n.value


def workspace_size(T: int, H: int, n_seqs: int, max_seqlen: int, dk: int = HEAD_DIM, dv: int = HEAD_DIM):
    """(bytes_min, bytes_full) of the prefill workspace."""
    lo, hi = ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = load_library().kda_chunk_fwd_workspace_size(T, H, dk, dv, n_seqs, max_seqlen, ctypes.byref(lo), ctypes.byref(hi))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_workspace_size")
    return lo.value, hi.value


def chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, *, cu_seqlens=None, max_seqlen=None,
              scale: float = 1.0, gate=None, norm_weight=None, eps: float = 1e-6, out_dtype=None,
              output_final_state: bool = True, final_state=None, out=None, workspace=None, stream=None,
              checkpoints=None, ckpt_tokens: int = 512, segments: int = 1):
    """Chunkwise KDA prefill.

    q, k, log_alpha: [B, T, H, 128]; v: [B, T, H, 128]; beta: [B, T, H] (bf16 or
    fp32, all the same dtype).  Varlen: B = 1 and cu_seqlens int32 [N+1] on the
    device plus max_seqlen (host int).  initial_state: fp32 [N, H, 128, 128] or
    None.  gate: [B, T, H, 128] or None (then o is returned unnormalised).
    Returns (o_or_y [B, T, H, 128], final_state fp32 [N, H, 128, 128] or None).
    checkpoints: None, True (allocate zeros) or fp32 [N, max_seqlen // ckpt_tokens, H, 128, 128]
    receiving the state after every ckpt_tokens tokens of each sequence (ckpt_tokens a
    multiple of 64); then the return value is (o, final_state, checkpoints).
    segments > 1: segment-parallel prefill (kda_chunk_fwd_segmented); not combined
    with checkpoints.
    """
    torch = _torch()
    _check_cuda(q, k, v, log_alpha, beta, initial_state, cu_seqlens, gate, norm_weight)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    in_dt = _dt(q)
    for t in (k, v, log_alpha, beta) + ((gate,) if gate is not None else ()):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, log_alpha, beta and gate must share one dtype")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        if max_seqlen is None:
            raise ValueError("varlen needs max_seqlen (host int)")
        N = cu_seqlens.numel() - 1
    else:
        N = B
        max_seqlen = T
    odt = out_dtype if out_dtype is not None else q.dtype
    o = out if out is not None else torch.empty((B, T, H, dv), dtype=odt, device=q.device)
    fs = final_state
    if fs is None and output_final_state:
        fs = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        if segments > 1:
            full = segmented_workspace_size(B * T if cu_seqlens is None else T, H, N, max_seqlen, segments, dk, dv)
        else:
            _, full = workspace_size(B * T if cu_seqlens is None else T, H, N, max_seqlen, dk, dv)
        workspace = torch.empty(full, dtype=torch.uint8, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state), _ptr(o), _ptr(fs),
            B, T, H, dk, dv, _ptr(cu_seqlens), N, int(max_seqlen), in_dt, _dt(o), float(scale), _ptr(gate),
            _ptr(norm_weight), float(eps))
    tail = (_ptr(workspace), workspace.numel(), _stream(stream))
    if segments > 1:
        if checkpoints is not None:
            raise ValueError("segments > 1 does not take checkpoints")
        st = load_library().kda_chunk_fwd_segmented(*args, int(segments), *tail)
        if st != KDA_OK:
            raise KdaError(st, "kda_chunk_fwd_segmented")
        return o, fs
    if checkpoints is None:
        st = load_library().kda_chunk_fwd(*args, *tail)
        if st != KDA_OK:
            raise KdaError(st, "kda_chunk_fwd")
        return o, fs
    if checkpoints is True:
        checkpoints = torch.zeros((N, int(max_seqlen) // ckpt_tokens, H, dk, dv), dtype=torch.float32,
                                  device=q.device)
    _check_cuda(checkpoints)
    st = load_library().kda_chunk_fwd_ckpt(*args, _ptr(checkpoints), int(ckpt_tokens), *tail)
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_ckpt")
    return o, fs, checkpoints


def bwd_workspace_size(T: int, H: int, n_seqs: int, max_seqlen: int, dk: int = HEAD_DIM, dv: int = HEAD_DIM) -> int:
    """Workspace bytes of chunk_bwd."""
    n = ctypes.c_size_t(0)
    st = load_library().kda_chunk_bwd_workspace_size(T, H, dk, dv, n_seqs, max_seqlen, ctypes.byref(n))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_bwd_workspace_size")
    return n.value


def chunk_bwd(q, k, v, log_alpha, beta, d_o, initial_state=None, d_final_state=None, *, cu_seqlens=None,
              max_seqlen=None, scale: float = 1.0, want_d_initial_state: bool = True, workspace=None, stream=None):
    """Gradients of chunk_fwd (no gate): inputs as chunk_fwd, d_o = dL/do [B, T, H, 128]
    (the inputs' dtype), d_final_state = dL/d(final state) fp32 [N, H, 128, 128] or None.
    Returns a dict of fp32 tensors: dq, dk, dv, dlog_alpha [B, T, H, 128], dbeta [B, T, H]
    and d_initial_state [N, H, 128, 128] (None when not wanted)."""
    torch = _torch()
    _check_cuda(q, k, v, log_alpha, beta, d_o, initial_state, d_final_state, cu_seqlens, workspace)
    B, T, N, maxlen = _seq_dims(q, cu_seqlens, max_seqlen)
    H, dk, dv = q.shape[2], q.shape[3], v.shape[-1]
    for t in (k, v, log_alpha, beta, d_o):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, log_alpha, beta and d_o must share one dtype")
    f32 = dict(dtype=torch.float32, device=q.device)
    g = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
             dv=torch.empty((B, T, H, dv), **f32), dlog_alpha=torch.empty((B, T, H, dk), **f32),
             dbeta=torch.empty((B, T, H), **f32),
             d_initial_state=torch.empty((N, H, dk, dv), **f32) if want_d_initial_state else None)
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B * T if cu_seqlens is None else T, H, N, maxlen, dk, dv),
                                dtype=torch.uint8, device=q.device)
    st = load_library().kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
                                      _ptr(d_o), _ptr(d_final_state), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                                      _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["d_initial_state"]), B, T, H,
                                      dk, dv, _ptr(cu_seqlens), N, maxlen, _dt(q), float(scale), _ptr(workspace),
                                      workspace.numel(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_bwd")
    return g


def _seq_dims(q, cu_seqlens, max_seqlen):
    torch = _torch()
    B, T = q.shape[0], q.shape[1]
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        if max_seqlen is None:
            raise ValueError("varlen needs max_seqlen (host int)")
        return B, T, cu_seqlens.numel() - 1, int(max_seqlen)
    return B, T, B, T


def kcp_workspace_size(T: int, H: int, n_seqs: int, max_seqlen: int, dk: int = HEAD_DIM, dv: int = HEAD_DIM) -> int:
    """Workspace bytes shared by kcp_transition and kcp_finish."""
    n = ctypes.c_size_t(0)
    st = load_library().kda_kcp_workspace_size(T, H, dk, dv, n_seqs, max_seqlen, ctypes.byref(n))
    if st != KDA_OK:
        raise KdaError(st, "kda_kcp_workspace_size")
    return n.value


def kcp_transition(q, k, v, log_alpha, beta, *, cu_seqlens=None, max_seqlen=None, scale: float = 1.0,
                   transition=None, workspace=None, stream=None):
    """Step 1 of context parallelism across devices, for this device's token
    segment (inputs as chunk_fwd).  Returns (transition fp32 [2, N, H, 128, 128]:
    [0] = M, [1] = B with S_out = M S_in + B; workspace holding the chunk work
    for kcp_finish)."""
    torch = _torch()
    _check_cuda(q, k, v, log_alpha, beta, cu_seqlens, transition, workspace)
    B, T, N, maxlen = _seq_dims(q, cu_seqlens, max_seqlen)
    H, dk, dv = q.shape[2], q.shape[3], v.shape[-1]
    for t in (k, v, log_alpha, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, log_alpha and beta must share one dtype")
    if transition is None:
        transition = torch.empty((2, N, H, dk, dk), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(kcp_workspace_size(B * T if cu_seqlens is None else T, H, N, maxlen, dk, dv),
                                dtype=torch.uint8, device=q.device)
    st = load_library().kda_kcp_transition(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), B, T, H, dk, dv,
                                           _ptr(cu_seqlens), N, maxlen, _dt(q), float(scale), _ptr(transition),
                                           _ptr(workspace), workspace.numel(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_kcp_transition")
    return transition, workspace


def kcp_compose(transitions, n_prev: int, initial_state=None, *, out=None, stream=None):
    """Step 3: folds maps 0 .. n_prev-1 of the gathered transitions
    ([R, 2, N, H, 128, 128] fp32, device order) over initial_state (fp32
    [N, H, 128, 128] or None = zero).  Returns this device's initial state."""
    torch = _torch()
    _check_cuda(transitions, initial_state, out)
    _, _, N, H, dk, dv = transitions.shape
    s_in = out if out is not None else torch.empty((N, H, dk, dv), dtype=torch.float32, device=transitions.device)
    st = load_library().kda_kcp_compose(_ptr(transitions), int(n_prev), _ptr(initial_state), _ptr(s_in), N, H, dk,
                                        dv, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_kcp_compose")
    return s_in


def kcp_finish(state_in, workspace, *, shape, dtype, cu_seqlens=None, max_seqlen=None, gate=None, norm_weight=None,
               eps: float = 1e-6, out_dtype=None, output_final_state: bool = True, out=None, stream=None):
    """Step 4: this device's outputs from its initial state and the workspace
    kcp_transition filled.  shape = (B, T, H, 128) and dtype of the segment's
    inputs (the gate's dtype).  Returns (o or y [B, T, H, 128], final_state)."""
    torch = _torch()
    _check_cuda(state_in, workspace, cu_seqlens, gate, norm_weight)
    B, T, H, dv = shape
    if gate is not None and gate.dtype != dtype:
        raise TypeError("the gate must have the inputs' dtype")
    if cu_seqlens is not None:
        if max_seqlen is None:
            raise ValueError("varlen needs max_seqlen (host int)")
        N, maxlen = cu_seqlens.numel() - 1, int(max_seqlen)
    else:
        N, maxlen = B, T
    in_dt = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    odt = out_dtype if out_dtype is not None else dtype
    o = out if out is not None else torch.empty((B, T, H, dv), dtype=odt, device=workspace.device)
    fs = torch.empty((N, H, HEAD_DIM, dv), dtype=torch.float32, device=workspace.device) if output_final_state else None
    st = load_library().kda_kcp_finish(_ptr(state_in), _ptr(o), _ptr(fs), B, T, H, HEAD_DIM, dv, _ptr(cu_seqlens), N,
                                       maxlen, in_dt, _dt(o), _ptr(gate), _ptr(norm_weight), float(eps),
                                       _ptr(workspace), workspace.numel(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_kcp_finish")
    return o, fs


def decode_step(state, q, k, v, log_alpha, beta, *, scale: float = 1.0, gate=None, norm_weight=None,
                eps: float = 1e-6, out_dtype=None, out=None, stream=None):
    """One recurrent step.  state: fp32 [Bd, H, 128, 128] (updated in place);
    q, k, log_alpha, v: [Bd, H, 128]; beta: [Bd, H].  Returns o (or y) [Bd, H, 128]."""
    torch = _torch()
    _check_cuda(state, q, k, v, log_alpha, beta, gate, norm_weight)
    if state.dtype != torch.float32:
        raise TypeError("state must be fp32")
    Bd, H, dk = q.shape
    dv = v.shape[-1]
    odt = out_dtype if out_dtype is not None else q.dtype
    o = out if out is not None else torch.empty((Bd, H, dv), dtype=odt, device=q.device)
    st = load_library().kda_decode_step(_ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(o),
                                        Bd, H, dk, dv, _dt(q), _dt(o), float(scale), _ptr(gate), _ptr(norm_weight),
                                        float(eps), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step")
    return o


def decode_steps(state, q, k, v, log_alpha, beta, *, scale: float = 1.0, gate=None, norm_weight=None,
                 eps: float = 1e-6, out_dtype=None, out=None, step_states=None, stream=None):
    """n consecutive recurrent steps in one call (e.g. verifying n draft tokens).
    state: fp32 [Bd, H, 128, 128], carried through the steps in place;
    q, k, log_alpha, v: [n, Bd, H, 128]; beta: [n, Bd, H].  step_states: None,
    True (allocate) or an fp32 [n, Bd, H, 128, 128] tensor that receives the state
    after every step.  Returns o (or y) [n, Bd, H, 128], or (o, step_states) when
    step_states was requested."""
    torch = _torch()
    want = step_states is not None
    if step_states is True:
        step_states = torch.empty((q.shape[0],) + tuple(state.shape), dtype=torch.float32, device=q.device)
    _check_cuda(state, q, k, v, log_alpha, beta, gate, norm_weight, step_states if want else None)
    if state.dtype != torch.float32:
        raise TypeError("state must be fp32")
    n, Bd, H, dk = q.shape
    dv = v.shape[-1]
    odt = out_dtype if out_dtype is not None else q.dtype
    o = out if out is not None else torch.empty((n, Bd, H, dv), dtype=odt, device=q.device)
    st = load_library().kda_decode_steps(_ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                         _ptr(o), n, Bd, H, dk, dv, _dt(q), _dt(o), float(scale), _ptr(gate),
                                         _ptr(norm_weight), float(eps), _ptr(step_states if want else None),
                                         _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_steps")
    return (o, step_states) if want else o


def gate_norm(o, g, norm_weight=None, *, eps: float = 1e-6, out_dtype=None, out=None, stream=None):
    """y = o / sqrt(mean(o^2) + eps) * w * sigmoid(g) over the last dim (128)."""
    torch = _torch()
    _check_cuda(o, g, norm_weight)
    dv = o.shape[-1]
    rows = o.numel() // dv
    odt = out_dtype if out_dtype is not None else o.dtype
    y = out if out is not None else torch.empty(o.shape, dtype=odt, device=o.device)
    st = load_library().kda_gate_norm(_ptr(o), _ptr(g), _ptr(norm_weight), float(eps), _ptr(y), rows, dv,
                                      _dt(o), _dt(y), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_gate_norm")
    return y


def query_status(workspace, stream=None) -> int:
    """Synchronises, returns and clears the device status word of a workspace."""
    return load_library().kda_query_status(_ptr(workspace), _stream(stream))


def profile_enable(on: bool = True) -> None:
    """Per-kernel device timing of later library launches (CUDA events)."""
    load_library().kda_profile_enable(int(bool(on)))


def profile_read() -> dict:
    """{kernel name: (launches, summed device ms)} since the last read."""
    arr = (KernelTime * 16)()
    n = ctypes.c_int(0)
    st = load_library().kda_profile_read(arr, 16, ctypes.byref(n))
    if st != KDA_OK:
        raise KdaError(st, "kda_profile_read")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].ms) for i in range(min(n.value, 16))}
