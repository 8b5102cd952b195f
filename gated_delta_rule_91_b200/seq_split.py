"""One sequence split across the ranks of a process group, in rank order.

Rank r owns tokens [r*T/R, (r+1)*T/R) of every (batch, head) -- any split
works, the segments only have to be consecutive and in rank order.  For one
(b, h) a segment maps the incoming state affinely, S_out = S_in M + N, and
its outputs are o_t = o_t(0) + S_in q~_t with q~_t = M_<=t q_t (the chunkwise
form of the Gated DeltaNet review, section 3.7, composed over the chunks of a
segment).  Per rank:

  1. gdr_seg_fwd on the local segment -> o(0), q~, N, M   (two forward passes)
  2. all-gather (M, N) of every rank                     (the one exchange)
  3. gdr_seg_combine -> this segment's S_in and the final state
  4. gdr_seg_fixup   -> o = o(0) + S_in q~

The exchange is B*H*(dk*dk + dv*dk) fp32 per rank (2 MiB for B1 H16 d128);
with NCCL it is one all-gather per tensor.  The arithmetic runs in the CUDA
library; this module only moves tensors between ranks.  `ops` replaces the
library calls (the CPU tests pass stand-ins; the product path never does).
"""
import torch
import torch.distributed as dist


class _LibOps:
    """The CUDA library's entry points (the product path)."""

    @staticmethod
    def seg_fwd(q, k, v, log_alpha, beta):
        from . import gdr_seg_fwd
        return gdr_seg_fwd(q, k, v, log_alpha, beta)

    @staticmethod
    def seg_combine(M_all, N_all, r, S0):
        from . import gdr_seg_combine
        return gdr_seg_combine(M_all, N_all, r, S0, want_final=True)

    @staticmethod
    def seg_fixup(qt, S_in, o):
        from . import gdr_seg_fixup
        return gdr_seg_fixup(qt, S_in, o)


def seq_split_fwd(q, k, v, log_alpha, beta, S0=None, *, group=None, ops=None):
    """Forward over this rank's segment of a sequence split across `group`.

    q, k [B,T_r,H,dk]; v [B,T_r,H,dv]; log_alpha, beta [B,T_r,H]: this rank's
    tokens.  S0 [B,H,dv,dk] fp32 (or None) is the state before the whole
    sequence and must be the same on every rank.  Returns (o [B,T_r,H,dv],
    S_T [B,H,dv,dk]): this segment's outputs and the state after the whole
    sequence (the same on every rank)."""
    ops = _LibOps if ops is None else ops
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    o, qt, N, M = ops.seg_fwd(q, k, v, log_alpha, beta)
    M_all = torch.empty((R,) + tuple(M.shape), dtype=M.dtype, device=M.device)
    N_all = torch.empty((R,) + tuple(N.shape), dtype=N.dtype, device=N.device)
    dist.all_gather(list(M_all.unbind(0)), M.contiguous(), group=group)
    dist.all_gather(list(N_all.unbind(0)), N.contiguous(), group=group)
    S_in, S_T = ops.seg_combine(M_all, N_all, r, S0)
    ops.seg_fixup(qt, S_in, o)
    return o, S_T
