"""Seeded synthetic inputs for the KDA workloads (input generation only).

Every tensor is produced by a counter-based generator (SplitMix64 in counter
mode, Box-Muller normals), so any token block of any tensor can be generated
on its own and equals the same block of the whole tensor.  Both the CUDA path's
tests/benchmark and the CPU oracle's tests draw their inputs from here; the
module holds none of the recurrence's arithmetic.

Distributions (token-major, head-minor layout [T, H, d]):
  q, k       N(0,1) per element, then each (token, head) row divided by its L2
             norm
  v          N(0,1)
  beta       sigmoid(N(0,1))                       [T, H]
  log_alpha  max(-5, -softplus(N(0,1)))            [T, H, dk]
  g (gate)   N(0,1)                                [T, H, dv]
  states     N(0, 0.02^2) fp32                     [N, H, dk, dv]
  lengths    integers uniform on [lo, hi], inclusive
With ``bf16=True`` every value is rounded to bf16 (round to nearest even) and
returned as the float32 holding that exact bf16 value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_synth.c")
_LIB = os.path.join(_HERE, "libkda_synth.so")

TAG_Q, TAG_K, TAG_V, TAG_BETA, TAG_LOG_ALPHA, TAG_GATE, TAG_STATE, TAG_LENGTHS = range(1, 9)
LOG_ALPHA_FLOOR = -5.0


def build(force: bool = False) -> str:
    """Compile the generator library in place (gcc) and return its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fvisibility=hidden",
               "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32p = ctypes.POINTER(ctypes.c_float)
        u64, i64, c_int, c_d = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.synth_normal.argtypes = [u64, u64, i64, i64, c_d, c_int, f32p]
        lib.synth_sigmoid_normal.argtypes = [u64, u64, i64, i64, c_int, f32p]
        lib.synth_neg_softplus_normal.argtypes = [u64, u64, i64, i64, c_d, c_int, f32p]
        lib.synth_unit_rows.argtypes = [u64, u64, i64, i64, c_int, c_int, f32p]
        lib.synth_unit_rows.restype = c_int
        lib.synth_uniform_int.argtypes = [u64, u64, i64, i64, i64, ctypes.POINTER(ctypes.c_int64)]
        lib.synth_to_bf16_bits.argtypes = [f32p, i64, ctypes.POINTER(ctypes.c_uint16)]
        _lib = lib
    return _lib


def _fp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def normal(seed: int, tag: int, shape, std: float = 1.0, bf16: bool = False, idx0: int = 0):
    out = np.empty(shape, dtype=np.float32)
    _L().synth_normal(seed, tag, idx0, out.size, std, int(bf16), _fp(out))
    return out


def unit_rows(seed: int, tag: int, shape, bf16: bool = False, row0: int = 0):
    """Rows along the last axis are N(0,1) vectors scaled to unit L2 norm."""
    out = np.empty(shape, dtype=np.float32)
    d = shape[-1]
    rc = _L().synth_unit_rows(seed, tag, row0, out.size // d, d, int(bf16), _fp(out))
    if rc != 0:
        raise ValueError("row length must be in [1, 1024]")
    return out


def sigmoid_normal(seed: int, tag: int, shape, bf16: bool = False, idx0: int = 0):
    out = np.empty(shape, dtype=np.float32)
    _L().synth_sigmoid_normal(seed, tag, idx0, out.size, int(bf16), _fp(out))
    return out


def neg_softplus_normal(seed: int, tag: int, shape, floor: float = LOG_ALPHA_FLOOR,
                        bf16: bool = False, idx0: int = 0):
    out = np.empty(shape, dtype=np.float32)
    _L().synth_neg_softplus_normal(seed, tag, idx0, out.size, floor, int(bf16), _fp(out))
    return out


def uniform_int(seed: int, tag: int, n: int, lo: int, hi: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    _L().synth_uniform_int(seed, tag, n, lo, hi, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    return out


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> uint16 bf16 bit patterns (round to nearest even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _L().synth_to_bf16_bits(_fp(a), a.size, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)))
    return out


@dataclass
class TokenBlock:
    """Per-token inputs for tokens [tok0, tok0+ntok) of a packed token stream."""
    q: np.ndarray          # [ntok, H, dk]
    k: np.ndarray          # [ntok, H, dk]
    v: np.ndarray          # [ntok, H, dv]
    log_alpha: np.ndarray  # [ntok, H, dk]
    beta: np.ndarray       # [ntok, H]
    g: np.ndarray | None   # [ntok, H, dv] (output gate) or None


def tokens(seed: int, tok0: int, ntok: int, H: int, dk: int, dv: int, bf16: bool,
           gate: bool = False) -> TokenBlock:
    """Inputs of tokens [tok0, tok0+ntok) of a packed stream with H heads."""
    rows = tok0 * H
    q = unit_rows(seed, TAG_Q, (ntok, H, dk), bf16, row0=rows)
    k = unit_rows(seed, TAG_K, (ntok, H, dk), bf16, row0=rows)
    v = normal(seed, TAG_V, (ntok, H, dv), 1.0, bf16, idx0=rows * dv)
    la = neg_softplus_normal(seed, TAG_LOG_ALPHA, (ntok, H, dk), LOG_ALPHA_FLOOR, bf16, idx0=rows * dk)
    beta = sigmoid_normal(seed, TAG_BETA, (ntok, H), bf16, idx0=rows)
    g = normal(seed, TAG_GATE, (ntok, H, dv), 1.0, bf16, idx0=rows * dv) if gate else None
    return TokenBlock(q, k, v, la, beta, g)


def states(seed: int, N: int, H: int, dk: int, dv: int, std: float = 0.02) -> np.ndarray:
    """fp32 states [N, H, dk, dv] with N(0, std^2) entries."""
    return normal(seed, TAG_STATE, (N, H, dk, dv), std, False)


def varlen_lengths(seed: int, n: int = 16, lo: int = 512, hi: int = 16384) -> np.ndarray:
    return uniform_int(seed, TAG_LENGTHS, n, lo, hi)


def cu_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu
