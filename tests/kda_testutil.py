"""Shared helpers for the parity tests: seeded inputs (from the synth module),
device upload, oracle runs and the error metric.

Tolerance (stated by the workload definition): relative L2 error
||x - x_ref||_2 / ||x_ref||_2 <= 1e-2 on outputs and on final states
(bf16 inputs, fp32 accumulation and state).
"""
from __future__ import annotations

import numpy as np

from linear_attention_recurrence_06_b200 import synth

REL_L2_TOL = 1e-2
D = 128


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    if den == 0.0:
        return float(num)
    return float(num / den)


def dev(a, dtype):
    """numpy float32 (already rounded to `dtype` where bf16) -> CUDA tensor."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device="cuda", dtype=dtype)


def host(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy()


def make_prefill(seed, lengths, H, bf16=True, gate=False, init=False, la_const=None, beta_const=None,
                 la_scale=None):
    """Packed varlen (or single) prefill inputs as numpy float32 arrays."""
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    tb = synth.tokens(seed, 0, T, H, D, D, bf16=bf16, gate=gate)
    la = tb.log_alpha
    if la_const is not None:
        la = np.full_like(la, la_const)
    if la_scale is not None:
        la = (la * la_scale).astype(np.float32)
        if bf16:
            la = ((synth.bf16_bits(la).astype(np.uint32) << 16).view(np.float32))
    beta = tb.beta if beta_const is None else np.full_like(tb.beta, beta_const)
    s0 = synth.states(seed, len(lengths), H, D, D) if init else None
    cu = synth.cu_from_lengths(lengths)
    return dict(q=tb.q, k=tb.k, v=tb.v, log_alpha=la, beta=beta, g=tb.g, s0=s0, cu=cu, T=T)


# Achieved errors of every parity comparison, printed at the end of the
# session (tests/conftest.py) so the margin to the tolerance is on record.
MARGINS = []


def assert_rel_l2(x, ref, what: str, tol: float = REL_L2_TOL) -> float:
    """Relative L2 error of x against ref, recorded with the running test's id,
    and asserted to be within tol."""
    import os
    e = rel_l2(x, ref)
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    MARGINS.append((test, what, e, tol))
    assert e <= tol, f"{what}: rel-L2 {e:.3e} above {tol:g}"
    return e


# Canary guard regions: an output buffer is allocated with GUARD extra elements
# on each side, all set to a fixed NaN bit pattern; after the call the guards
# must still hold it (a cheap stand-in for an out-of-bounds write checker).
GUARD = 1024
_CANARY = {"float32": (0x7FC0DEAD, "int32"), "bfloat16": (0x7FDE, "int16")}


def guarded_empty(shape, dtype):
    """(tensor of `shape` on the GPU, check()) where check() asserts that
    nothing was written into the guard regions around it."""
    import torch
    n = int(np.prod(shape))
    pat, ity = _CANARY[str(dtype).split(".")[-1]]
    ity = getattr(torch, ity)
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    buf.view(ity).fill_(pat)
    inner = buf[GUARD:GUARD + n].view(shape)

    def check(what="output"):
        torch.cuda.synchronize()
        for side, part in (("before", buf[:GUARD]), ("after", buf[GUARD + n:])):
            bad = (part.view(ity) != pat).nonzero()
            assert bad.numel() == 0, f"{what}: {bad.numel()} guard elements {side} the buffer were overwritten"
    return inner, check
