"""Device-side failure paths, exercised without faulting the GPU.

* cu_seqlens that contradict T or max_seqlen: the kernels clamp every sequence
  range into [0, T] and walk at most max_seqlen / 64 chunks per sequence, so no
  access leaves the buffers; a check kernel records the contradiction in the
  workspace status word, and kda_query_status returns KDA_ERR_DEVICE_ARG.
* A bounded wait that gives up: a test hook makes one CTA of the chunk-local
  kernel skip one of its first tile loads, so the transaction count its barrier
  waits for is never reached; with the wait limit shortened to 2 ms the CTA gives
  up, records KDA_ERR_TIMEOUT and leaves through its normal exit (TMEM freed).
Both times the next call in the same process is normal and matches the oracle.
"""
import numpy as np
import pytest

import oracle
from kda_testutil import D, assert_rel_l2, dev, guarded_empty, host, make_prefill

pytestmark = pytest.mark.gpu

KDA_ERR_TIMEOUT, KDA_ERR_DEVICE_ARG = -6, -7


def _inputs(seed, lens, H):
    import torch
    inp = make_prefill(seed, lens, H, bf16=True, init=True)
    T = inp["T"]
    t = {x: dev(inp[x], torch.bfloat16).view(1, T, H, D) for x in ("q", "k", "v", "log_alpha")}
    t["beta"] = dev(inp["beta"], torch.bfloat16).view(1, T, H)
    t["s0"] = dev(inp["s0"], torch.float32)
    return inp, t


def _clean_call_matches_oracle(kda, inp, t, lens, H, ws):
    import torch
    T = inp["T"]
    cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
    o, o_check = guarded_empty((1, T, H, D), torch.float32)
    fs, fs_check = guarded_empty((len(lens), H, D, D), torch.float32)
    kda.chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["s0"], cu_seqlens=cu, max_seqlen=max(lens),
                  out=o, final_state=fs, workspace=ws)
    assert kda.query_status(ws) == 0
    o_check("o")
    fs_check("final state")
    ro, rfs = oracle.kda_recurrent(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["s0"], inp["cu"])
    assert_rel_l2(host(o).reshape(T, H, D), ro, "o after the failed call")
    assert_rel_l2(host(fs), rfs, "final state after the failed call")


@pytest.mark.parametrize("case", ["longer_than_max_seqlen", "last_offset_short_of_T", "last_offset_past_T",
                                  "decreasing"])
def test_seqlen_contradiction_is_reported(case):
    import torch
    import linear_attention_recurrence_06_b200 as kda
    lens, H = [100, 200, 37], 2
    inp, t = _inputs(131, lens, H)
    T = inp["T"]
    cu = inp["cu"].astype(np.int32).copy()
    max_seqlen = max(lens)
    if case == "longer_than_max_seqlen":
        max_seqlen = 128        # sequence 1 has 200 tokens
    elif case == "last_offset_short_of_T":
        cu[-1] = T - 5
    elif case == "last_offset_past_T":
        cu[-1] = T + 50          # clamped to T by the kernels
    else:
        cu[2] = cu[1] - 10       # sequence 1 has a negative length (empty once clamped)
    _, full = kda.workspace_size(T, H, len(lens), max(lens))
    ws = torch.empty(full, dtype=torch.uint8, device="cuda")
    o, o_check = guarded_empty((1, T, H, D), torch.float32)
    fs, fs_check = guarded_empty((len(lens), H, D, D), torch.float32)
    kda.chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["s0"],
                  cu_seqlens=torch.from_numpy(cu).cuda(), max_seqlen=max_seqlen, out=o, final_state=fs,
                  workspace=ws)
    assert kda.query_status(ws) == KDA_ERR_DEVICE_ARG
    o_check("o")
    fs_check("final state")
    assert kda.query_status(ws) == 0  # reading the word cleared it
    _clean_call_matches_oracle(kda, inp, t, lens, H, ws)


def test_wait_that_gives_up_is_reported():
    import torch
    import linear_attention_recurrence_06_b200 as kda
    lib = kda.load_library()
    lens, H = [300, 129], 2
    inp, t = _inputs(137, lens, H)
    T = inp["T"]
    cu = torch.from_numpy(inp["cu"].astype(np.int32)).cuda()
    _, full = kda.workspace_size(T, H, len(lens), max(lens))
    ws = torch.empty(full, dtype=torch.uint8, device="cuda")
    assert lib.kda_test_drop_tile_load(2_000_000) == 0
    try:
        kda.chunk_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["s0"], cu_seqlens=cu,
                      max_seqlen=max(lens), workspace=ws)
    finally:
        lib.kda_test_drop_tile_load(0)  # never leave the hook pending for another test
    assert kda.query_status(ws) == KDA_ERR_TIMEOUT
    _clean_call_matches_oracle(kda, inp, t, lens, H, ws)
