"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and the CPU-baseline leg of bench.py may
import this package.  It shares no code with the CUDA library and the product
path never reaches it.

The arithmetic lives in gdr_oracle.c (plain sequential recurrences in double
precision, one token at a time).  This module only marshals numpy float64
arrays into that library.  Parity of each function is pinned by the
tests/test_oracle_*.py files.
"""
import ctypes
import os

import numpy as np

from .build import build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.oracle_gdr_fwd.argtypes = [i, i, i, i, i] + [dp] * 8
        lib.oracle_gdr_step.argtypes = [i, i, i, i] + [dp] * 7
        lib.oracle_gdr_bwd.argtypes = [i, i, i, i, i] + [dp] * 14
        lib.oracle_gdr2_fwd.argtypes = [i, i, i, i, i] + [dp] * 9
        lib.oracle_gdr2_bwd.argtypes = [i, i, i, i, i] + [dp] * 16
        lib.oracle_short_conv.argtypes = [i] * 5 + [dp] * 4 + [i, ctypes.c_double, dp, dp]
        lib.oracle_rmsnorm_gate.argtypes = [i] * 4 + [dp] * 3 + [ctypes.c_double, dp]
        lib.oracle_rmsnorm_gate_bwd.argtypes = [i] * 4 + [dp] * 3 + [ctypes.c_double] + [dp] * 4
        lib.oracle_short_conv_bwd.argtypes = [i] * 5 + [dp] * 4 + [i, ctypes.c_double] + [dp] * 6
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _in(x):
    if x is None:
        return None
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    """Host threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def gdr_fwd(q, k, v, log_alpha, beta, S0=None):
    """Sequential gated delta rule forward.  Shapes: q,k [B,T,H,dk],
    v [B,T,H,dv], log_alpha/beta [B,T,H], S0 [B,H,dv,dk] or None.
    Returns (o [B,T,H,dv], S_T [B,H,dv,dk]) as float64."""
    q, k, v, la, be, S0 = map(_in, (q, k, v, log_alpha, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    _load().oracle_gdr_fwd(B, T, H, dk, dv, _p(q), _p(k), _p(v), _p(la), _p(be),
                           _p(S0), _p(o), _p(ST))
    return o, ST


def gdr_step(q, k, v, log_alpha, beta, S):
    """One decode token.  q,k [B,H,dk], v [B,H,dv], log_alpha/beta [B,H],
    S [B,H,dv,dk].  Returns (o [B,H,dv], S_new) without modifying S."""
    q, k, v, la, be = map(_in, (q, k, v, log_alpha, beta))
    S = np.array(S, dtype=np.float64, copy=True, order="C")
    B, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, dv))
    _load().oracle_gdr_step(B, H, dk, dv, _p(q), _p(k), _p(v), _p(la), _p(be),
                            _p(S), _p(o))
    return o, S


def gdr_step_inplace(q, k, v, log_alpha, beta, S):
    """One decode token applied to S in place (S: float64, C-contiguous
    [B,H,dv,dk], as returned by an earlier call or built by the caller).
    Returns o [B,H,dv].  Same arithmetic as gdr_step without the copy of S,
    for long decode sequences over a large state."""
    q, k, v, la, be = map(_in, (q, k, v, log_alpha, beta))
    if S.dtype != np.float64 or not S.flags["C_CONTIGUOUS"]:
        raise ValueError("S must be a C-contiguous float64 array")
    B, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, dv))
    _load().oracle_gdr_step(B, H, dk, dv, _p(q), _p(k), _p(v), _p(la), _p(be),
                            _p(S), _p(o))
    return o


def gdr_bwd(q, k, v, log_alpha, beta, S0, dO, dS_T=None):
    """Hand-derived reverse mode of gdr_fwd.  Returns a dict with dq, dk, dv,
    dlog_alpha, dbeta, dS0 (float64)."""
    q, k, v, la, be, S0, dO, dST = map(_in, (q, k, v, log_alpha, beta, S0, dO, dS_T))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dlog_alpha=np.zeros_like(la), dbeta=np.zeros_like(be),
               dS0=np.zeros((B, H, dv, dk)))
    _load().oracle_gdr_bwd(B, T, H, dk, dv, _p(q), _p(k), _p(v), _p(la), _p(be),
                           _p(S0), _p(dO), _p(dST), _p(out["dq"]), _p(out["dk"]),
                           _p(out["dv"]), _p(out["dlog_alpha"]), _p(out["dbeta"]),
                           _p(out["dS0"]))
    return out


def gdr2_fwd(q, k, v, log_alpha, b, w, S0=None):
    """Gated Delta Rule-2 forward.  log_alpha, b [B,T,H,dk]; w [B,T,H,dv].
    Returns (o, S_T) as float64."""
    q, k, v, la, bb, ww, S0 = map(_in, (q, k, v, log_alpha, b, w, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    _load().oracle_gdr2_fwd(B, T, H, dk, dv, _p(q), _p(k), _p(v), _p(la), _p(bb),
                            _p(ww), _p(S0), _p(o), _p(ST))
    return o, ST


def gdr2_bwd(q, k, v, log_alpha, b, w, S0, dO, dS_T=None):
    """Hand-derived reverse mode of gdr2_fwd.  Returns a dict with dq, dk, dv,
    dlog_alpha, db, dw, dS0 (float64)."""
    q, k, v, la, bb, ww, S0, dO, dST = map(_in, (q, k, v, log_alpha, b, w, S0, dO, dS_T))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dlog_alpha=np.zeros_like(la), db=np.zeros_like(bb), dw=np.zeros_like(ww),
               dS0=np.zeros((B, H, dv, dk)))
    _load().oracle_gdr2_bwd(B, T, H, dk, dv, _p(q), _p(k), _p(v), _p(la), _p(bb), _p(ww),
                            _p(S0), _p(dO), _p(dST), _p(out["dq"]), _p(out["dk"]),
                            _p(out["dv"]), _p(out["dlog_alpha"]), _p(out["db"]), _p(out["dw"]),
                            _p(out["dS0"]))
    return out


def short_conv(x, w, bias=None, state=None, l2=False, eps=0.0):
    """Block prologue for one stream: depthwise causal ShortConv of width K,
    SiLU, and (l2=True) L2 normalisation per (token, head).  x [B,T,H,d],
    w [H*d, K], bias [H*d] or None, state [B, K-1, H*d] or None (zeros).
    Returns (y [B,T,H,d], state_out [B, K-1, H*d]) as float64."""
    x, w, bias, state = map(_in, (x, w, bias, state))
    B, T, H, d = x.shape
    K = w.shape[-1]
    y = np.zeros_like(x)
    st = np.zeros((B, K - 1, H * d))
    _load().oracle_short_conv(B, T, H, d, K, _p(x), _p(w), _p(bias), _p(state), int(l2),
                              float(eps), _p(y), _p(st) if K > 1 else None)
    return y, st


def short_conv_bwd(x, w, dy, bias=None, state=None, dstate_out=None, l2=False, eps=0.0):
    """Reverse mode of short_conv for an incoming dy [B,T,H,d] (and the
    gradient of the returned state, dstate_out [B,K-1,H*d], or None).
    Returns dict(dx [B,T,H,d], dw [H*d,K], dbias [H*d], dstate [B,K-1,H*d])."""
    x, w, dy, bias, state, dso = map(_in, (x, w, dy, bias, state, dstate_out))
    B, T, H, d = x.shape
    K = w.shape[-1]
    out = dict(dx=np.zeros_like(x), dw=np.zeros((H * d, K)), dbias=np.zeros(H * d),
               dstate=np.zeros((B, K - 1, H * d)))
    _load().oracle_short_conv_bwd(B, T, H, d, K, _p(x), _p(w), _p(bias), _p(state), int(l2), float(eps),
                                  _p(dy), _p(dso) if K > 1 else None, _p(out["dx"]), _p(out["dw"]),
                                  _p(out["dbias"]), _p(out["dstate"]) if K > 1 else None)
    return out


def rmsnorm_gate(o, g, weight, eps=0.0):
    """Block epilogue: RMSNorm over dv per (token, head) with a per-channel
    weight, times SiLU(g) (g None: no gate).  o, g [B,T,H,dv], weight [dv]."""
    o, g, weight = map(_in, (o, g, weight))
    B, T, H, dv = o.shape
    y = np.zeros_like(o)
    _load().oracle_rmsnorm_gate(B, T, H, dv, _p(o), _p(g), _p(weight), float(eps), _p(y))
    return y


def rmsnorm_gate_bwd(o, g, weight, dy, eps=0.0):
    """Reverse mode of rmsnorm_gate: returns dict(do, dg (None without a
    gate), dweight [dv])."""
    o, g, weight, dy = map(_in, (o, g, weight, dy))
    B, T, H, dv = o.shape
    out = dict(do=np.zeros_like(o), dg=None if g is None else np.zeros_like(o), dweight=np.zeros(dv))
    _load().oracle_rmsnorm_gate_bwd(B, T, H, dv, _p(o), _p(g), _p(weight), float(eps), _p(dy),
                                    _p(out["do"]), _p(out["dg"]), _p(out["dweight"]))
    return out
