"""torch.autograd bindings of the library's forward/backward pairs.

`gated_delta_rule(q, k, v, log_alpha, beta, S0=None)` returns (o, S_T) and
differentiates through gdr_bwd; `gated_delta_rule2(q, k, v, log_alpha, b, w,
S0=None)` does the same for Gated DeltaNet-2 through gdr2_bwd.  The forward
and the backward are the library's CUDA calls: these classes only save the
inputs and hand the incoming gradients over (the backward recomputes the
forward's states itself, so nothing else is kept).  Unused outputs arrive as
zero gradients.  `block_prologue(...)` (ShortConv, SiLU, q/k L2) and
`block_epilogue(o, g, weight, eps)` (RMSNorm, weight, SiLU gate) are the
block's steps around the recurrence, differentiated through
gdr_block_prologue_bwd and gdr_block_epilogue_bwd.
"""
import torch

from . import (gdr2_bwd, gdr2_fwd, gdr_block_epilogue, gdr_block_epilogue_bwd, gdr_block_prologue,
               gdr_block_prologue_bwd, gdr_bwd, gdr_fwd)


def _c(x):
    return None if x is None else x.contiguous()


class GatedDeltaRule(torch.autograd.Function):
    """o_t = S_t q_t with S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T."""

    @staticmethod
    def forward(ctx, q, k, v, log_alpha, beta, S0):
        q, k, v, log_alpha, beta, S0 = map(_c, (q, k, v, log_alpha, beta, S0))
        o, S_T = gdr_fwd(q, k, v, log_alpha, beta, S0)
        ctx.save_for_backward(q, k, v, log_alpha, beta, S0)
        return o, S_T

    @staticmethod
    def backward(ctx, dO, dS_T):
        q, k, v, log_alpha, beta, S0 = ctx.saved_tensors
        g = gdr_bwd(q, k, v, log_alpha, beta, S0, _c(dO), _c(dS_T), want_dS0=S0 is not None)
        return g["dq"], g["dk"], g["dv"], g["dlog_alpha"], g["dbeta"], g["dS0"]


class GatedDeltaRule2(torch.autograd.Function):
    """Gated Delta Rule-2: per-channel decay alpha, erase gate b, write gate w."""

    @staticmethod
    def forward(ctx, q, k, v, log_alpha, b, w, S0):
        q, k, v, log_alpha, b, w, S0 = map(_c, (q, k, v, log_alpha, b, w, S0))
        o, S_T = gdr2_fwd(q, k, v, log_alpha, b, w, S0)
        ctx.save_for_backward(q, k, v, log_alpha, b, w, S0)
        return o, S_T

    @staticmethod
    def backward(ctx, dO, dS_T):
        q, k, v, log_alpha, b, w, S0 = ctx.saved_tensors
        g = gdr2_bwd(q, k, v, log_alpha, b, w, S0, _c(dO), _c(dS_T), want_dS0=S0 is not None)
        return g["dq"], g["dk"], g["dv"], g["dlog_alpha"], g["db"], g["dw"], g["dS0"]


def gated_delta_rule(q, k, v, log_alpha, beta, S0=None):
    """Differentiable gdr_fwd: returns (o, S_T)."""
    return GatedDeltaRule.apply(q, k, v, log_alpha, beta, S0)


def gated_delta_rule2(q, k, v, log_alpha, b, w, S0=None):
    """Differentiable gdr2_fwd: returns (o, S_T)."""
    return GatedDeltaRule2.apply(q, k, v, log_alpha, b, w, S0)


class BlockEpilogue(torch.autograd.Function):
    """y = RMSNorm(o) * weight * SiLU(g) over dv per (token, head)."""

    @staticmethod
    def forward(ctx, o, g, weight, eps):
        o, g = _c(o), _c(g)
        ctx.eps = eps
        ctx.save_for_backward(o, g, weight)
        return gdr_block_epilogue(o, g, weight, eps)

    @staticmethod
    def backward(ctx, dy):
        o, g, weight = ctx.saved_tensors
        do, dg, dweight = gdr_block_epilogue_bwd(o, g, weight, _c(dy), ctx.eps)
        return do, dg, dweight, None


def block_epilogue(o, g, weight, eps=1e-6):
    """Differentiable gdr_block_epilogue: returns y."""
    return BlockEpilogue.apply(o, g, weight, eps)


class BlockPrologue(torch.autograd.Function):
    """q = L2(SiLU(conv(xq))), k = L2(SiLU(conv(xk))), v = SiLU(conv(xv)),
    the convolution reading the carried conv state before token 0."""

    @staticmethod
    def forward(ctx, xq, xk, xv, wq, wk, wv, bq, bk, bv, conv_state, eps):
        xq, xk, xv, conv_state = map(_c, (xq, xk, xv, conv_state))
        ctx.eps = eps
        ctx.has_bias = bq is not None
        ctx.save_for_backward(xq, xk, xv, wq, wk, wv, bq, bk, bv, conv_state)
        return gdr_block_prologue(xq, xk, xv, wq, wk, wv, bq, bk, bv, conv_state=conv_state, eps=eps)

    @staticmethod
    def backward(ctx, dq, dk, dv):
        xq, xk, xv, wq, wk, wv, bq, bk, bv, conv_state = ctx.saved_tensors
        g = gdr_block_prologue_bwd(xq, xk, xv, wq, wk, wv, _c(dq), _c(dk), _c(dv), bq, bk, bv,
                                   conv_state=conv_state, eps=ctx.eps, want_dbias=ctx.has_bias,
                                   want_dconv_state=conv_state is not None)
        return (g["dxq"], g["dxk"], g["dxv"], g["dwq"], g["dwk"], g["dwv"], g["dbq"], g["dbk"], g["dbv"],
                g["dconv_state"], None)


def block_prologue(xq, xk, xv, wq, wk, wv, bq=None, bk=None, bv=None, conv_state=None, eps=1e-6):
    """Differentiable gdr_block_prologue: returns (q, k, v)."""
    return BlockPrologue.apply(xq, xk, xv, wq, wk, wv, bq, bk, bv, conv_state, eps)
