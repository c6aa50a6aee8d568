"""kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot
allocate device memory (hosts that give a plugin only its inputs and outputs).
Its scratch is a static array inside the library, so the call takes no
workspace.  Called here through the C ABI (ctypes on libkda.so) and compared
with kda_chunk_fwd on the same inputs, on two calls in a row (the second call
finds the first call's leftovers in the shared array).

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest

from kda_testutil import REL_L2_TOL, D, dev, host, make_prefill, rel_l2

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 * 1024 * 1024


def _noalloc_fn():
    import linear_attention_recurrence_06_b200 as kda
    lib = kda.load_library()
    f = lib.kda_chunk_fwd_noalloc
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    f.restype = i32
    f.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, vp, i32, i64, i32, i32, f32, vp, vp, f32,
                  vp]
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_chunk_fwd_twice():
    import torch
    import linear_attention_recurrence_06_b200 as kda
    f = _noalloc_fn()
    lens = [300, 77, 129]
    H = 4
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((21, 22)):
        inp = make_prefill(seed, lens, H, bf16=True, init=True, gate=True)
        T = inp["T"]
        dt = torch.bfloat16
        q, k, v, la, g = (dev(inp[x], dt).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha", "g"))
        b = dev(inp["beta"], dt).view(1, T, H)
        s0 = dev(inp["s0"], torch.float32)
        cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
        mx = max(lens)
        ref_o, ref_s = kda.chunk_fwd(q, k, v, la, b, s0, cu_seqlens=cu, max_seqlen=mx, gate=g,
                                     out_dtype=torch.float32)
        o = torch.empty((1, T, H, D), dtype=torch.float32, device="cuda")
        s = torch.empty_like(ref_s)
        st = f(_p(q), _p(k), _p(v), _p(la), _p(b), _p(s0), _p(o), _p(s), 1, T, H, D, D, _p(cu), len(lens), mx,
               kda.KDA_BF16, kda.KDA_F32, 1.0, _p(g), None, 1e-6, stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert rel_l2(host(o), host(ref_o)) <= REL_L2_TOL
        assert rel_l2(host(s), host(ref_s)) <= REL_L2_TOL


def test_noalloc_rejects_problems_beyond_the_scratch():
    import linear_attention_recurrence_06_b200 as kda
    f = _noalloc_fn()
    fake = ctypes.c_void_p(0x10000)
    # 64 sequences x 32 heads needs far more than the static scratch
    lo, _ = kda.workspace_size(64 * 128, 32, 64, 128)
    assert lo > SCRATCH_BYTES
    st = f(fake, fake, fake, fake, fake, None, fake, fake, 64, 128, 32, D, D, None, 0, 128, kda.KDA_BF16,
           kda.KDA_BF16, 1.0, None, None, 1e-6, None)
    assert st == -4  # KDA_ERR_WORKSPACE, before any CUDA call
