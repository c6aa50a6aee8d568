"""The C-ABI library loads without a GPU, exports every entry point that
include/kda.h declares, and rejects bad arguments on the host before any
launch (these calls never reach CUDA)."""
import ctypes
import os
import re

import pytest

import linear_attention_recurrence_06_b200 as kda
from linear_attention_recurrence_06_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("kda_chunk_fwd", "kda_chunk_fwd_ckpt", "kda_chunk_fwd_segmented", "kda_decode_step", "kda_decode_steps",
              "kda_gate_norm", "kda_chunk_fwd_segmented_workspace_size",
              "kda_chunk_fwd_workspace_size", "kda_kcp_workspace_size", "kda_kcp_transition", "kda_kcp_compose",
              "kda_kcp_finish", "kda_chunk_bwd", "kda_chunk_bwd_workspace_size",
              "kda_query_status", "kda_status_string", "kda_version", "kda_chunk_fwd_noalloc",
              "kda_chunk_fwd_noalloc_query_status", "kda_test_drop_tile_load"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib, s), s


def test_status_strings(lib):
    for st in range(0, -8, -1):
        assert lib.kda_status_string(st).decode().startswith("KDA_")
    assert lib.kda_version() >= 100


def test_workspace_size(lib):
    lo, hi = kda.workspace_size(8192, 32, 1, 8192)
    assert 0 < lo <= hi
    # 128 chunks of one sequence
    per_slot = 32768 + 16384 + 32768 + 16384 + 512
    assert hi - lo == 127 * 32 * per_slot
    lo2, hi2 = kda.workspace_size(100, 2, 3, 50)
    assert hi2 >= lo2
    with pytest.raises(kda.KdaError):
        kda.workspace_size(100, 2, 3, 50, dk=64)


FAKE = 0x10000  # never dereferenced: every call below is rejected on the host


def _chunk(lib, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, o=FAKE, fs=None, B=1, T=128, H=2, dk=128,
                dv=128, cu=None, N=1, maxlen=128, idt=1, odt=1, scale=1.0, gate=None, w=None, eps=1e-6,
                ws=FAKE, wsb=1 << 40, stream=None)
    args.update(over)
    a = args
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["o"], a["fs"], a["B"], a["T"],
                             a["H"], a["dk"], a["dv"], a["cu"], a["N"], a["maxlen"], a["idt"], a["odt"], a["scale"],
                             a["gate"], a["w"], a["eps"], a["ws"], a["wsb"], a["stream"])


def test_chunk_fwd_ckpt_host_validation(lib):
    def ck(ptr, every, **over):
        args = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, o=FAKE, fs=None, B=1, T=128, H=2,
                    dk=128, dv=128, cu=None, N=1, maxlen=128, idt=1, odt=1, scale=1.0, gate=None, w=None, eps=1e-6,
                    ws=FAKE, wsb=1 << 40, stream=None)
        args.update(over)
        a = args
        return lib.kda_chunk_fwd_ckpt(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["o"], a["fs"], a["B"],
                                      a["T"], a["H"], a["dk"], a["dv"], a["cu"], a["N"], a["maxlen"], a["idt"],
                                      a["odt"], a["scale"], a["gate"], a["w"], a["eps"], ptr, every, a["ws"],
                                      a["wsb"], a["stream"])
    assert ck(FAKE, 100) == -1      # not a multiple of the chunk length
    assert ck(FAKE, 0) == -1
    assert ck(FAKE + 4, 64) == -3   # misaligned checkpoint buffer
    assert ck(FAKE, 64, q=None) == -1


def test_segmented_workspace_size(lib):
    import ctypes
    plain_lo, plain_full = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(4096, 4, 128, 128, 2, 2048, ctypes.byref(plain_lo),
                                            ctypes.byref(plain_full)) == 0
    seg = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_segmented_workspace_size(4096, 4, 128, 128, 2, 2048, 8, ctypes.byref(seg)) == 0
    assert seg.value == plain_full.value + 2 * 8 * 4 * 98816  # every chunk plus one map per segment
    assert lib.kda_chunk_fwd_segmented_workspace_size(4096, 4, 128, 128, 2, 2048, 1, ctypes.byref(seg)) == 0
    assert seg.value == plain_full.value
    assert lib.kda_chunk_fwd_segmented_workspace_size(4096, 4, 128, 128, 2, 2048, 0, ctypes.byref(seg)) == -1


def test_kcp_workspace_and_host_validation(lib):
    import ctypes
    full = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(4096, 4, 128, 128, 2, 2048, None, ctypes.byref(full)) == 0
    n = ctypes.c_size_t(0)
    assert lib.kda_kcp_workspace_size(4096, 4, 128, 128, 2, 2048, ctypes.byref(n)) == 0
    assert n.value == full.value  # both halves share every chunk's slot
    assert lib.kda_kcp_workspace_size(4096, 4, 128, 128, 2, 2048, None) == -1

    def tr(**over):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, B=1, T=128, H=2, dk=128, dv=128, cu=None, N=1,
                 maxlen=128, idt=1, scale=1.0, trans=FAKE, ws=FAKE, wsb=1 << 40)
        a.update(over)
        return lib.kda_kcp_transition(a["q"], a["k"], a["v"], a["la"], a["beta"], a["B"], a["T"], a["H"], a["dk"],
                                      a["dv"], a["cu"], a["N"], a["maxlen"], a["idt"], a["scale"], a["trans"],
                                      a["ws"], a["wsb"], None)
    assert tr(trans=None) == -1
    assert tr(k=None) == -1
    assert tr(trans=FAKE + 4) == -3
    assert tr(dk=64) == -2
    assert tr(H=70000) == -2
    assert tr(wsb=1024) == -4
    # the whole-sequence workspace is required (no multi-pass form)
    lo, hi = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(128, 2, 128, 128, 1, 128, ctypes.byref(lo), ctypes.byref(hi)) == 0
    assert tr(wsb=hi.value - 1) == -4

    def fin(**over):
        a = dict(s_in=None, o=FAKE, fs=None, B=1, T=128, H=2, dk=128, dv=128, cu=None, N=1, maxlen=128, idt=1,
                 odt=1, gate=None, w=None, eps=1e-6, ws=FAKE, wsb=1 << 40)
        a.update(over)
        return lib.kda_kcp_finish(a["s_in"], a["o"], a["fs"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["cu"],
                                  a["N"], a["maxlen"], a["idt"], a["odt"], a["gate"], a["w"], a["eps"], a["ws"],
                                  a["wsb"], None)
    assert fin(o=None) == -1
    assert fin(s_in=FAKE + 8) == -3
    assert fin(ws=None) == -4
    assert fin(eps=-1.0) == -1
    assert fin(cu=FAKE, B=2, N=2) == -1
    # compose: negative count, missing maps, misaligned buffers, unsupported dims
    assert lib.kda_kcp_compose(FAKE, -1, None, FAKE, 1, 2, 128, 128, None) == -1
    assert lib.kda_kcp_compose(None, 2, None, FAKE, 1, 2, 128, 128, None) == -1
    assert lib.kda_kcp_compose(FAKE, 2, None, None, 1, 2, 128, 128, None) == -1
    assert lib.kda_kcp_compose(FAKE, 2, FAKE + 4, FAKE, 1, 2, 128, 128, None) == -3
    assert lib.kda_kcp_compose(FAKE, 2, None, FAKE, 1, 2, 64, 128, None) == -2


def test_chunk_bwd_workspace_and_host_validation(lib):
    import ctypes
    full = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(300, 2, 128, 128, 1, 300, None, ctypes.byref(full)) == 0
    n = ctypes.c_size_t(0)
    assert lib.kda_chunk_bwd_workspace_size(300, 2, 128, 128, 1, 300, ctypes.byref(n)) == 0
    # the forward's whole-sequence workspace + 5 chunk-end gradients + 4 chunk-boundary states,
    # each a bf16 128 x 128 image per head
    assert n.value == full.value + (5 + 4) * 2 * 128 * 128 * 2

    def bw(**over):
        a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, s0=None, do=FAKE, dfin=None, dq=FAKE, dk=FAKE,
                 dv=FAKE, dla=FAKE, db=FAKE, dinit=None, B=1, T=128, H=2, dk_=128, dv_=128, cu=None, N=1,
                 maxlen=128, idt=1, scale=1.0, ws=FAKE, wsb=1 << 40)
        a.update(over)
        return lib.kda_chunk_bwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["s0"], a["do"], a["dfin"], a["dq"],
                                 a["dk"], a["dv"], a["dla"], a["db"], a["dinit"], a["B"], a["T"], a["H"], a["dk_"],
                                 a["dv_"], a["cu"], a["N"], a["maxlen"], a["idt"], a["scale"], a["ws"], a["wsb"],
                                 None)
    assert bw(do=None) == -1
    assert bw(dla=None) == -1
    assert bw(db=None) == -1
    assert bw(idt=5) == -1
    assert bw(dk_=64) == -2
    assert bw(H=70000) == -2
    assert bw(dq=FAKE + 4) == -3
    assert bw(dinit=FAKE + 8) == -3
    assert bw(ws=FAKE + 16) == -3
    assert bw(ws=None) == -4
    assert bw(wsb=1024) == -4
    assert bw(cu=FAKE, B=2, N=2) == -1


def test_chunk_fwd_host_validation(lib):
    assert _chunk(lib, q=None) == -1
    assert _chunk(lib, o=None) == -1
    assert _chunk(lib, H=0) == -1
    assert _chunk(lib, idt=7) == -1
    assert _chunk(lib, dk=64) == -2
    assert _chunk(lib, dv=256) == -2
    assert _chunk(lib, k=FAKE + 8) == -3
    assert _chunk(lib, ws=FAKE + 16) == -3      # workspace needs 256-byte alignment
    assert _chunk(lib, ws=None) == -4
    assert _chunk(lib, wsb=1024) == -4
    assert _chunk(lib, cu=FAKE, B=2, N=2) == -1  # varlen needs B = 1
    assert _chunk(lib, cu=FAKE, N=0) == -1
    assert _chunk(lib, cu=FAKE, N=2, maxlen=129) == -1  # longer than T
    assert _chunk(lib, eps=-1.0) == -1


def test_decode_and_gate_norm_host_validation(lib):
    assert lib.kda_decode_step(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 128, 1, 1, 1.0, None, None,
                               1e-6, None) == -1
    assert lib.kda_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 128, 1, 1, 1.0, None, None,
                               1e-6, None) == -2
    assert lib.kda_decode_step(FAKE, FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 128, 128, 1, 1, 1.0, None,
                               None, 1e-6, None) == -3
    assert lib.kda_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2, 128, 128, 1, 1, 1.0, None, None,
                               1e-6, None) == 0  # nothing to do, no launch
    # multi-step decode: negative step count, misaligned step_states, nothing to do
    assert lib.kda_decode_steps(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, -1, 4, 2, 128, 128, 1, 1, 1.0, None, None,
                                1e-6, None, None) == -1
    assert lib.kda_decode_steps(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 3, 4, 2, 128, 128, 1, 1, 1.0, None, None,
                                1e-6, FAKE + 8, None) == -3
    assert lib.kda_decode_steps(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 2, 128, 128, 1, 1, 1.0, None, None,
                                1e-6, None, None) == 0
    assert lib.kda_gate_norm(FAKE, FAKE, None, 1e-6, FAKE, -1, 128, 1, 1, None) == -1
    assert lib.kda_gate_norm(FAKE, FAKE, None, 1e-6, FAKE, 10, 64, 1, 1, None) == -2
    assert lib.kda_gate_norm(FAKE, FAKE, None, 1e-6, FAKE, 10, 128, 1, 0, None) == -1  # in place, sizes differ
    assert lib.kda_query_status(None, None) == -1


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 128)
    with pytest.raises(ValueError):
        kda.chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


def test_failure_hooks_host_side(lib):
    """The test hook that makes one tile load go missing takes a wait limit in
    [1 us, 1 s] (0 cancels a pending drop); other values are rejected on the
    host.  Setting and cancelling it touch no device."""
    assert lib.kda_test_drop_tile_load(5) == -1
    assert lib.kda_test_drop_tile_load(2_000_000_000) == -1
    assert lib.kda_test_drop_tile_load(2_000_000) == 0
    assert lib.kda_test_drop_tile_load(0) == 0  # cancelled again


def test_build_tracks_every_header(tmp_path):
    """An edit to any header the CUDA sources include (the slot layout among
    them) makes the library out of date, so it is rebuilt before use."""
    hs = [os.path.basename(h) for h in kbuild.headers()]
    for name in ("kda_slots.h", "kda_launch.h", "kda_profile.h", "kda_sm100.cuh", "kda.h"):
        assert name in hs, name
    kbuild.build()
    assert kbuild.up_to_date()
    slots = os.path.join(kbuild.CSRC, "kda_slots.h")
    st = os.stat(slots)
    lib_t = os.path.getmtime(kbuild.LIB)
    try:
        os.utime(slots, (st.st_atime, lib_t + 10))
        assert not kbuild.up_to_date()
    finally:
        os.utime(slots, (st.st_atime, st.st_mtime))
    assert kbuild.up_to_date()


# The boundary's entry points as declared in include/kda.h.  Against the planned boundary
# (the scope table's list: kda_chunk_fwd(q, k, v, log_alpha, beta, init_state -> o,
# final_state; B, T, H, dk, dv, cu_seqlens ...), kda_decode_step, kda_gate_norm,
# kda_query_status, kda_chunk_fwd_workspace_size, kda_status_string) the differences are
# deliberate: kda_chunk_fwd takes max_seqlen (the host never reads cu_seqlens), the
# workspace query returns a minimum and a full size (multi-pass workspaces), kda_decode_step
# takes the optional fused gate, kda_status_string takes an int (callable from any
# language), and streams pass as void*.  Pinning the declarations here makes any further
# change to them a visible, reviewed edit.
BOUNDARY = {
    "kda_chunk_fwd": ("kda_status", [
        "const void* q", "const void* k", "const void* v", "const void* log_alpha", "const void* beta",
        "const float* init_state", "void* o", "float* final_state", "int B", "int64_t T", "int H", "int dk",
        "int dv", "const int32_t* cu_seqlens", "int n_seqs", "int64_t max_seqlen", "kda_dtype in_dtype",
        "kda_dtype out_dtype", "float scale", "const void* gate", "const float* norm_weight", "float eps",
        "void* workspace", "size_t workspace_bytes", "void* stream"]),
    "kda_decode_step": ("kda_status", [
        "float* state", "const void* q", "const void* k", "const void* v", "const void* log_alpha",
        "const void* beta", "void* o", "int Bd", "int H", "int dk", "int dv", "kda_dtype in_dtype",
        "kda_dtype out_dtype", "float scale", "const void* gate", "const float* norm_weight", "float eps",
        "void* stream"]),
    "kda_gate_norm": ("kda_status", [
        "const void* o", "const void* gate", "const float* norm_weight", "float eps", "void* y", "int64_t rows",
        "int dv", "kda_dtype in_dtype", "kda_dtype out_dtype", "void* stream"]),
    "kda_query_status": ("kda_status", ["void* workspace", "void* stream"]),
    "kda_chunk_fwd_workspace_size": ("kda_status", [
        "int64_t T", "int H", "int dk", "int dv", "int n_seqs", "int64_t max_seqlen", "size_t* bytes_min",
        "size_t* bytes_full"]),
    "kda_status_string": ("const char*", ["int status"]),
}


def test_boundary_declarations_are_pinned():
    txt = open(HEADER).read()
    for name, (ret, params) in BOUNDARY.items():
        m = re.search(r"KDA_API\s+([\w\s\*]+?)\b" + name + r"\s*\(([^;]*?)\);", txt, re.S)
        assert m, name
        assert " ".join(m.group(1).split()) == ret, name
        assert [" ".join(p.split()) for p in m.group(2).split(",")] == params, name
