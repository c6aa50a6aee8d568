"""Context parallelism across devices (KCP) for sequences longer than one GPU
should walk alone.

Sources: the nlpx.cn K3 paper walkthrough, §6 (KCP: the recurrence split over
devices through segment transitions), and the "training and inference systems"
item of the K3 article summaries on the xhh.club tag page (context parallelism
as a prefix scan of segment transitions).

One process per GPU.  Rank r of ``group`` holds token segment r of every
sequence (consecutive segments in rank order).  A segment acts on the state as
the affine map S -> M_r S + B_r, so the ranks need one exchange:

  1. transition  each rank runs the chunk-local kernels over its segment, keeps
                 their output in its workspace and produces (M_r, B_r) fp32
                 (``kcp_transition``);
  2. all-gather  of the maps, 2 * N * H * 128 * 128 fp32 per rank (4 MiB at N = 1,
                 H = 32), over NCCL (NVLink / NVSwitch on one node);
  3. compose     rank r folds maps 0 .. r-1 over the sequences' initial state
                 (``kcp_compose``, one small kernel);
  4. finish      rank r walks its kept chunks from that state with outputs
                 (``kcp_finish``).

The per-rank steps go through a backend object so that the exchange and the
ordering logic here can be exercised on CPU ranks (gloo) with other per-rank
implementations; the default backend is the CUDA library.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass
class SegmentArgs:
    """Shape facts of this rank's segment that the finish step needs."""
    shape: tuple
    dtype: object
    cu_seqlens: object = None
    max_seqlen: int | None = None


class CudaBackend:
    """The per-rank steps on the CUDA library (the product path)."""

    def transition(self, q, k, v, log_alpha, beta, *, scale, cu_seqlens, max_seqlen, stream=None):
        from . import kcp_transition
        trans, ws = kcp_transition(q, k, v, log_alpha, beta, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen,
                                   scale=scale, stream=stream)
        return trans, (ws, SegmentArgs(tuple(q.shape[:3]) + (v.shape[-1],), q.dtype, cu_seqlens, max_seqlen))

    def compose(self, gathered, n_prev, initial_state, stream=None):
        from . import kcp_compose
        return kcp_compose(gathered, n_prev, initial_state, stream=stream)

    def finish(self, state_in, ctx, *, gate, norm_weight, eps, out_dtype, stream=None):
        from . import kcp_finish
        ws, seg = ctx
        return kcp_finish(state_in, ws, shape=seg.shape, dtype=seg.dtype, cu_seqlens=seg.cu_seqlens,
                          max_seqlen=seg.max_seqlen, gate=gate, norm_weight=norm_weight, eps=eps,
                          out_dtype=out_dtype, stream=stream)


def gather_transitions(trans, group=None):
    """All-gather of every rank's maps in rank order: [R, 2, N, H, dk, dk]."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = trans.new_empty((world,) + tuple(trans.shape))
    # concatenation along dim 0 is the layout both NCCL and gloo gather into
    dist.all_gather_into_tensor(out.view((world * trans.shape[0],) + tuple(trans.shape[1:])), trans.contiguous(),
                                group=group)
    return out


def kcp_prefill(q, k, v, log_alpha, beta, initial_state=None, *, group=None, scale: float = 1.0, gate=None,
                norm_weight=None, eps: float = 1e-6, out_dtype=None, cu_seqlens=None, max_seqlen=None,
                backend=None, stream=None):
    """This rank's part of a prefill whose sequences are split over the ranks
    of ``group`` (rank r holds segment r).  Inputs as ``chunk_fwd`` for the
    local segment; ``initial_state`` is the sequences' state before segment 0
    and must be the same on every rank (or None everywhere).  Returns
    (o or y of the local tokens, state after the local segment); the last
    rank's state is the sequences' final state."""
    import torch.distributed as dist
    be = backend if backend is not None else CudaBackend()
    rank = dist.get_rank(group)
    trans, ctx = be.transition(q, k, v, log_alpha, beta, scale=scale, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen,
                               stream=stream)
    if stream is not None and getattr(trans, "is_cuda", False):
        import torch
        with torch.cuda.stream(stream):  # the collective follows the kernels on their stream
            gathered = gather_transitions(trans, group)
    else:
        gathered = gather_transitions(trans, group)
    state_in = be.compose(gathered, rank, initial_state, stream=stream)
    return be.finish(state_in, ctx, gate=gate, norm_weight=norm_weight, eps=eps, out_dtype=out_dtype, stream=stream)
