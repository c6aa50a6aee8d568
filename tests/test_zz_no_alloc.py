"""kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot
allocate device memory (hosts that give a plugin only its inputs and outputs,
or forbid cudaMalloc on their hot path because it can synchronise the device).
Its scratch is a static array inside the library, so the call takes no
workspace.  Called here through the C ABI (ctypes on libkda.so) and compared
with kda_chunk_fwd on the same inputs and with the fp64 oracle, on two calls
in a row (the second call finds the first call's leftovers in the shared
array); the device status word of the array is read back through
kda_chunk_fwd_noalloc_query_status.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest

import oracle
from kda_testutil import D, assert_rel_l2, dev, guarded_empty, host, make_prefill

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 * 1024 * 1024


def _lib():
    import linear_attention_recurrence_06_b200 as kda
    return kda.load_library()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(lib, t, o, s, cu, n_seqs, T, H, max_seqlen, stream):
    import linear_attention_recurrence_06_b200 as kda
    return lib.kda_chunk_fwd_noalloc(_p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["la"]), _p(t["b"]), _p(t["s0"]),
                                     _p(o), _p(s), 1, T, H, D, D, _p(cu), n_seqs, max_seqlen, kda.KDA_BF16,
                                     kda.KDA_F32, 1.0, _p(t["g"]), None, 1e-6, stream)


def _inputs(seed, lens, H):
    import torch
    inp = make_prefill(seed, lens, H, bf16=True, init=True, gate=True)
    T = inp["T"]
    dt = torch.bfloat16
    t = {n: dev(inp[x], dt).view(1, T, H, D) for n, x in (("q", "q"), ("k", "k"), ("v", "v"), ("la", "log_alpha"),
                                                          ("g", "g"))}
    t["b"] = dev(inp["beta"], dt).view(1, T, H)
    t["s0"] = dev(inp["s0"], torch.float32)
    return inp, t


def test_noalloc_matches_chunk_fwd_and_oracle_twice():
    import torch
    import linear_attention_recurrence_06_b200 as kda
    lib = _lib()
    lens = [300, 77, 129]
    H = 4
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((21, 22)):
        inp, t = _inputs(seed, lens, H)
        T = inp["T"]
        cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
        mx = max(lens)
        ref_o, ref_s = kda.chunk_fwd(t["q"], t["k"], t["v"], t["la"], t["b"], t["s0"], cu_seqlens=cu, max_seqlen=mx,
                                     gate=t["g"], out_dtype=torch.float32)
        o, o_check = guarded_empty((1, T, H, D), torch.float32)
        s, s_check = guarded_empty(tuple(ref_s.shape), torch.float32)
        st = _call(lib, t, o, s, cu, len(lens), T, H, mx, stream)
        assert st == 0, f"call {call}: status {st}"
        assert lib.kda_chunk_fwd_noalloc_query_status(stream) == 0
        o_check(f"call {call} y")
        s_check(f"call {call} final state")
        # the existing entry point on the same inputs
        assert_rel_l2(host(o), host(ref_o), f"call {call} y against kda_chunk_fwd")
        assert_rel_l2(host(s), host(ref_s), f"call {call} final state against kda_chunk_fwd")
        # and the fp64 oracle
        ro, rfs = oracle.kda_recurrent(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["s0"],
                                       inp["cu"])
        ry = oracle.gate_norm(ro, inp["g"], None, 1e-6)
        assert_rel_l2(host(o).reshape(T, H, D), ry, f"call {call} y against the oracle")
        assert_rel_l2(host(s), rfs, f"call {call} final state against the oracle")


def test_noalloc_reports_device_errors():
    """cu_seqlens with a sequence longer than max_seqlen: the kernels stay in
    bounds (ranges are clamped), the status word in the static array records the
    contradiction and the companion query returns KDA_ERR_DEVICE_ARG; the next
    clean call reports KDA_OK."""
    import torch
    lib = _lib()
    lens, H = [200, 64], 2
    inp, t = _inputs(23, lens, H)
    T = inp["T"]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
    o = torch.empty((1, T, H, D), dtype=torch.float32, device="cuda")
    s = torch.empty((len(lens), H, D, D), dtype=torch.float32, device="cuda")
    assert _call(lib, t, o, s, cu, len(lens), T, H, 128, stream) == 0  # sequence 0 has 200 > 128 tokens
    assert lib.kda_chunk_fwd_noalloc_query_status(stream) == -7       # KDA_ERR_DEVICE_ARG
    assert lib.kda_chunk_fwd_noalloc_query_status(stream) == 0        # the query cleared it
    assert _call(lib, t, o, s, cu, len(lens), T, H, max(lens), stream) == 0
    assert lib.kda_chunk_fwd_noalloc_query_status(stream) == 0


def test_noalloc_rejects_problems_beyond_the_scratch():
    import linear_attention_recurrence_06_b200 as kda
    lib = _lib()
    fake = ctypes.c_void_p(0x10000)
    # 64 sequences x 32 heads needs far more than the static scratch
    lo, _ = kda.workspace_size(64 * 128, 32, 64, 128)
    assert lo > SCRATCH_BYTES
    st = lib.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, None, fake, fake, 64, 128, 32, D, D, None, 0, 128,
                                   kda.KDA_BF16, kda.KDA_BF16, 1.0, None, None, 1e-6, None)
    assert st == -4  # KDA_ERR_WORKSPACE, before any CUDA call
