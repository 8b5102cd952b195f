"""Python binding of libgdr.so, the B200 (sm_100a) gated delta rule library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/gdr.h.  PyTorch supplies device
memory (outputs, workspace) and the current CUDA stream.  There is no CPU
path: if libgdr.so is missing or no GPU is present the calls raise.

Functions (same names as the C entry points):
    gdr_fwd(q, k, v, log_alpha, beta, S0=None)          -> (o, S_T)
    gdr_step(q, k, v, log_alpha, beta, S)                -> o  (S advanced in place)
    gdr_bwd(q, k, v, log_alpha, beta, S0, dO, dS_T=None) -> dict of gradients
    gdr2_fwd(q, k, v, log_alpha, b, w, S0=None)          -> (o, S_T)
    gdr2_bwd(q, k, v, log_alpha, b, w, S0, dO, dS_T=None) -> dict of gradients
    gdr2_step(q, k, v, log_alpha, b, w, S)               -> o  (S advanced in place)
    gdr_block_prologue(xq, xk, xv, wq, wk, wv, ...)       -> (q, k, v)
    gdr_block_prologue_bwd(xq, xk, xv, wq, wk, wv, dq, dk, dv, ...) -> dict of gradients
    gdr_block_epilogue(o, g, weight, eps)                 -> y
    gdr_block_epilogue_bwd(o, g, weight, dy, eps)         -> (do, dg, dweight)
    gdr_seg_fwd / gdr_seg_combine / gdr_seg_fixup         (sequence split; see seq_split)

The calls take the current CUDA stream and allocate nothing inside the
library, so they can be captured in CUDA graphs.  `autograd` wraps the
forward/backward pairs as torch.autograd Functions.
"""
import ctypes
import os

import torch

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libgdr.so")

GDR_OK, GDR_ERR_INVALID_ARGUMENT, GDR_ERR_UNSUPPORTED, GDR_ERR_WORKSPACE, GDR_ERR_CUDA, \
    GDR_ERR_TIMEOUT = range(6)
GDR_F32, GDR_BF16 = 0, 1
STATUS_NAMES = {0: "GDR_OK", 1: "GDR_ERR_INVALID_ARGUMENT", 2: "GDR_ERR_UNSUPPORTED",
                3: "GDR_ERR_WORKSPACE", 4: "GDR_ERR_CUDA", 5: "GDR_ERR_TIMEOUT"}

# name -> (restype, argtypes); mirrors include/gdr.h
_I, _SZ, _P = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
SIGNATURES = {
    "gdr_fwd": (_I, [_I] * 6 + [_P] * 8 + [_P, _SZ, _P]),
    "gdr_fwd_workspace_bytes": (_SZ, [_I] * 6),
    "gdr_step": (_I, [_I] * 5 + [_P] * 7 + [_P]),
    "gdr_bwd": (_I, [_I] * 6 + [_P] * 14 + [_P, _SZ, _P]),
    "gdr_bwd_workspace_bytes": (_SZ, [_I] * 6),
    "gdr_bwd_noalloc": (_I, [_I] * 6 + [_P] * 14 + [_P]),
    "gdr2_fwd": (_I, [_I] * 6 + [_P] * 9 + [_P, _SZ, _P]),
    "gdr2_fwd_workspace_bytes": (_SZ, [_I] * 6),
    "gdr2_bwd": (_I, [_I] * 6 + [_P] * 16 + [_P, _SZ, _P]),
    "gdr2_bwd_workspace_bytes": (_SZ, [_I] * 6),
    "gdr2_step": (_I, [_I] * 5 + [_P] * 8 + [_P]),
    "gdr_block_prologue": (_I, [_I] * 7 + [_P] * 11 + [ctypes.c_float] + [_P] * 3 + [_P]),
    "gdr_block_prologue_bwd": (_I, [_I] * 7 + [_P] * 10 + [ctypes.c_float] + [_P] * 14 + [_P, _SZ, _P]),
    "gdr_block_prologue_bwd_workspace_bytes": (_SZ, [_I] * 4),
    "gdr_block_epilogue": (_I, [_I] * 5 + [_P] * 3 + [ctypes.c_float, _P, _P]),
    "gdr_block_epilogue_bwd": (_I, [_I] * 5 + [_P] * 3 + [ctypes.c_float] + [_P] * 5 + [_SZ, _P]),
    "gdr_block_epilogue_bwd_workspace_bytes": (_SZ, [_I]),
    "gdr_seg_fwd": (_I, [_I] * 6 + [_P] * 9 + [_P, _SZ, _P]),
    "gdr_seg_fwd_workspace_bytes": (_SZ, [_I] * 6),
    "gdr_seg_combine": (_I, [_I] * 6 + [_P] * 5 + [_P]),
    "gdr_seg_fixup": (_I, [_I] * 6 + [_P] * 3 + [_P]),
    "gdr_check_status": (_I, [_P]),
    "gdr_debug_wait_timeout": (_I, [_I, _P]),
    "gdr_last_error_string": (ctypes.c_char_p, []),
    "gdr_launch_count": (ctypes.c_uint64, []),
    "gdr_version": (_I, []),
}


class GdrError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), msg))
        self.status = status


_lib = None


def lib():
    """The loaded libgdr.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libgdr.so not found at %s; build it with "
                               "`python -m gated_delta_rule_91_b200._build`" % LIB_PATH)
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def check(status):
    if status != GDR_OK:
        raise GdrError(status, lib().gdr_last_error_string().decode())


def launch_count() -> int:
    return int(lib().gdr_launch_count())


def check_status(stream=None):
    """Synchronise the stream and raise if a kernel recorded a timeout."""
    s = torch.cuda.current_stream() if stream is None else stream
    check(lib().gdr_check_status(ctypes.c_void_p(s.cuda_stream)))


def _dt(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return GDR_F32
    if x.dtype == torch.bfloat16:
        return GDR_BF16
    raise TypeError("q/k/v must be float32 or bfloat16, got %s" % x.dtype)


def _ptr(x):
    if x is None:
        return None
    if not x.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not x.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(x.data_ptr())


def _f32(x, name):
    if x is not None and x.dtype != torch.float32:
        raise TypeError("%s must be float32" % name)
    return x


def _stream(x):
    return ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream)


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def gdr_fwd(q, k, v, log_alpha, beta, S0=None, *, o=None, S_T=None, return_state=True,
            workspace=None):
    """Chunkwise forward on the current stream.  Returns (o, S_T or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    _f32(log_alpha, "log_alpha"), _f32(beta, "beta"), _f32(S0, "S0")
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    if S_T is None and return_state:
        S_T = torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device)
    L = lib()
    ws, ws_bytes = _workspace(L.gdr_fwd_workspace_bytes(B, T, H, dk, dv, dt), q.device, workspace)
    check(L.gdr_fwd(B, T, H, dk, dv, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                    _ptr(S0), _ptr(o), _ptr(S_T), _ptr(ws), ws_bytes, _stream(q)))
    return o, S_T


def gdr_step(q, k, v, log_alpha, beta, S, *, o=None):
    """One decode token; S [B,H,dv,dk] fp32 is advanced in place.  Returns o."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    _f32(S, "S")
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    check(lib().gdr_step(B, H, dk, dv, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                         _ptr(beta), _ptr(S), _ptr(o), _stream(q)))
    return o


def gdr_bwd(q, k, v, log_alpha, beta, S0, dO, dS_T=None, *, want_dS0=True, workspace=None):
    """Backward of gdr_fwd.  Returns dict(dq, dk, dv, dlog_alpha, dbeta, dS0)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dlog_alpha=torch.empty_like(log_alpha), dbeta=torch.empty_like(beta),
               dS0=torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device)
               if want_dS0 else None)
    L = lib()
    ws, ws_bytes = _workspace(L.gdr_bwd_workspace_bytes(B, T, H, dk, dv, dt), q.device, workspace)
    check(L.gdr_bwd(B, T, H, dk, dv, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                    _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]),
                    _ptr(out["dv"]), _ptr(out["dlog_alpha"]), _ptr(out["dbeta"]),
                    _ptr(out["dS0"]), _ptr(ws), ws_bytes, _stream(q)))
    return out


def gdr2_fwd(q, k, v, log_alpha, b, w, S0=None, *, o=None, S_T=None, return_state=True,
             workspace=None):
    """Gated DeltaNet-2 forward.  Returns (o, S_T or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    if S_T is None and return_state:
        S_T = torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device)
    L = lib()
    ws, ws_bytes = _workspace(L.gdr2_fwd_workspace_bytes(B, T, H, dk, dv, dt), q.device, workspace)
    check(L.gdr2_fwd(B, T, H, dk, dv, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b),
                     _ptr(w), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(ws), ws_bytes, _stream(q)))
    return o, S_T


def gdr2_step(q, k, v, log_alpha, b, w, S, *, o=None):
    """One Gated DeltaNet-2 decode token.  q, k [B,H,dk]; v [B,H,dv];
    log_alpha, b [B,H,dk] fp32; w [B,H,dv] fp32; S [B,H,dv,dk] fp32 updated in
    place.  Returns o [B,H,dv]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    _f32(log_alpha, "log_alpha"), _f32(b, "b"), _f32(w, "w"), _f32(S, "S")
    if o is None:
        o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    check(lib().gdr2_step(B, H, dk, dv, _dt(q), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                          _ptr(S), _ptr(o), _stream(q)))
    return o


def gdr2_bwd(q, k, v, log_alpha, b, w, S0, dO, dS_T=None, *, want_dS0=True, workspace=None):
    """Backward of gdr2_fwd.  Returns dict(dq, dk, dv, dlog_alpha, db, dw, dS0)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dlog_alpha=torch.empty_like(log_alpha), db=torch.empty_like(b), dw=torch.empty_like(w),
               dS0=torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device) if want_dS0 else None)
    L = lib()
    ws, ws_bytes = _workspace(L.gdr2_bwd_workspace_bytes(B, T, H, dk, dv, dt), q.device, workspace)
    check(L.gdr2_bwd(B, T, H, dk, dv, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                     _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                     _ptr(out["dlog_alpha"]), _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dS0"]),
                     _ptr(ws), ws_bytes, _stream(q)))
    return out


def gdr_block_prologue(xq, xk, xv, wq, wk, wv, bq=None, bk=None, bv=None, *, conv_state=None,
                       conv_state_out=None, eps=1e-6, q=None, k=None, v=None):
    """The block's q/k/v paths after the input projections: depthwise causal
    ShortConv (taps w* [H*d, K] fp32, biases b* [H*d] or None), SiLU, and L2
    normalisation of q and k per (token, head).  xq, xk [B,T,H,dk]; xv
    [B,T,H,dv].  conv_state [B, K-1, H*(2dk+dv)] (dtype of x, channels q, k,
    v) carries the inputs before token 0; conv_state_out receives the last
    K-1 inputs and may be conv_state itself.  Returns (q, k, v)."""
    B, T, H, dk = xq.shape
    dv = xv.shape[-1]
    K = wq.shape[-1]
    dt = _dt(xq)
    for name, t in (("wq", wq), ("wk", wk), ("wv", wv), ("bq", bq), ("bk", bk), ("bv", bv)):
        _f32(t, name)
    q = torch.empty_like(xq) if q is None else q
    k = torch.empty_like(xk) if k is None else k
    v = torch.empty_like(xv) if v is None else v
    check(lib().gdr_block_prologue(B, T, H, dk, dv, K, dt, _ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq),
                                   _ptr(wk), _ptr(wv), _ptr(bq), _ptr(bk), _ptr(bv),
                                   _ptr(conv_state), _ptr(conv_state_out), float(eps), _ptr(q),
                                   _ptr(k), _ptr(v), _stream(xq)))
    return q, k, v


def gdr_block_prologue_bwd(xq, xk, xv, wq, wk, wv, dyq, dyk, dyv, bq=None, bk=None, bv=None, *,
                           conv_state=None, dconv_state_out=None, eps=1e-6, want_dbias=None,
                           want_dconv_state=None, workspace=None):
    """Backward of gdr_block_prologue for incoming gradients dyq, dyk, dyv of
    (q, k, v) and optionally of the returned conv state.  Returns dict(dxq,
    dxk, dxv, dwq, dwk, dwv, dbq, dbk, dbv (None unless a bias was given or
    want_dbias), dconv_state (None unless conv_state was given or
    want_dconv_state))."""
    B, T, H, dk = xq.shape
    dv = xv.shape[-1]
    K = wq.shape[-1]
    for n, t in (("wq", wq), ("wk", wk), ("wv", wv), ("bq", bq), ("bk", bk), ("bv", bv)):
        _f32(t, n)
    want_db = (bq is not None) if want_dbias is None else want_dbias
    want_ds = (conv_state is not None) if want_dconv_state is None else want_dconv_state
    out = dict(dxq=torch.empty_like(xq), dxk=torch.empty_like(xk), dxv=torch.empty_like(xv))
    for n, t in (("dwq", wq), ("dwk", wk), ("dwv", wv)):
        out[n] = torch.empty_like(t)
    for n, d in (("dbq", dk), ("dbk", dk), ("dbv", dv)):
        out[n] = torch.empty(H * d, dtype=torch.float32, device=xq.device) if want_db else None
    out["dconv_state"] = (torch.empty(B, max(K - 1, 0), H * (2 * dk + dv), dtype=xq.dtype, device=xq.device)
                          if want_ds and K > 1 else None)
    L = lib()
    ws, ws_bytes = _workspace(L.gdr_block_prologue_bwd_workspace_bytes(H, dk, dv, K), xq.device, workspace)
    check(L.gdr_block_prologue_bwd(
        B, T, H, dk, dv, K, _dt(xq), _ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(bq),
        _ptr(bk), _ptr(bv), _ptr(conv_state), float(eps), _ptr(dyq), _ptr(dyk), _ptr(dyv), _ptr(dconv_state_out),
        _ptr(out["dxq"]), _ptr(out["dxk"]), _ptr(out["dxv"]), _ptr(out["dwq"]), _ptr(out["dwk"]),
        _ptr(out["dwv"]), _ptr(out["dbq"]), _ptr(out["dbk"]), _ptr(out["dbv"]), _ptr(out["dconv_state"]),
        _ptr(ws), ws_bytes, _stream(xq)))
    return out


def gdr_block_epilogue(o, g, weight, eps=1e-6, *, y=None):
    """RMSNorm of the recurrent output over dv per (token, head), times the
    per-channel weight [dv] fp32 and SiLU(g) (g None: no gate).  o, g
    [B,T,H,dv].  Returns y."""
    B, T, H, dv = o.shape
    _f32(weight, "weight")
    y = torch.empty_like(o) if y is None else y
    check(lib().gdr_block_epilogue(B, T, H, dv, _dt(o), _ptr(o), _ptr(g), _ptr(weight), float(eps),
                                   _ptr(y), _stream(o)))
    return y


def gdr_block_epilogue_bwd(o, g, weight, dy, eps=1e-6, *, workspace=None):
    """Backward of gdr_block_epilogue for an incoming dy [B,T,H,dv]: returns
    (do, dg or None without a gate, dweight [dv] fp32)."""
    B, T, H, dv = o.shape
    _f32(weight, "weight")
    do = torch.empty_like(o)
    dg = None if g is None else torch.empty_like(g)
    dweight = torch.empty(dv, dtype=torch.float32, device=o.device)
    L = lib()
    ws, ws_bytes = _workspace(L.gdr_block_epilogue_bwd_workspace_bytes(dv), o.device, workspace)
    check(L.gdr_block_epilogue_bwd(B, T, H, dv, _dt(o), _ptr(o), _ptr(g), _ptr(weight), float(eps), _ptr(dy),
                                   _ptr(do), _ptr(dg), _ptr(dweight), _ptr(ws), ws_bytes, _stream(o)))
    return do, dg, dweight


def gdr_seg_fwd(q, k, v, log_alpha, beta, *, workspace=None):
    """Both forward passes of one segment of a split sequence: returns
    (o0 [B,T,H,dv] from S_in = 0, qt [B,T,H,dk] = M_<=t q_t,
     N [B,H,dv,dk], M [B,H,dk,dk])."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    o0 = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    qt = torch.empty(B, T, H, dk, dtype=q.dtype, device=q.device)
    N = torch.empty(B, H, dv, dk, dtype=torch.float32, device=q.device)
    M = torch.empty(B, H, dk, dk, dtype=torch.float32, device=q.device)
    L = lib()
    ws, ws_bytes = _workspace(L.gdr_seg_fwd_workspace_bytes(B, T, H, dk, dv, dt), q.device, workspace)
    check(L.gdr_seg_fwd(B, T, H, dk, dv, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                        _ptr(o0), _ptr(qt), _ptr(N), _ptr(M), _ptr(ws), ws_bytes, _stream(q)))
    return o0, qt, N, M


def gdr_seg_combine(M_all, N_all, r, S0=None, *, want_final=True):
    """Sequential combine of the segment maps: M_all [R,B,H,dk,dk], N_all
    [R,B,H,dv,dk] in segment order.  Returns (S_in of segment r, state after
    the last segment or None)."""
    R, B, H, dk, _ = M_all.shape
    dv = N_all.shape[3]
    _f32(M_all, "M_all"), _f32(N_all, "N_all"), _f32(S0, "S0")
    S_in = torch.empty(B, H, dv, dk, dtype=torch.float32, device=M_all.device)
    S_T = torch.empty_like(S_in) if want_final else None
    check(lib().gdr_seg_combine(R, r, B, H, dk, dv, _ptr(M_all), _ptr(N_all), _ptr(S0), _ptr(S_in),
                                _ptr(S_T), _stream(M_all)))
    return S_in, S_T


def gdr_seg_fixup(qt, S_in, o):
    """o += S_in q~ per token (in place); returns o."""
    B, T, H, dk = qt.shape
    dv = o.shape[-1]
    _f32(S_in, "S_in")
    check(lib().gdr_seg_fixup(B, T, H, dk, dv, _dt(qt), _ptr(qt), _ptr(S_in), _ptr(o), _stream(qt)))
    return o
