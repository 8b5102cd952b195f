"""The C-ABI library loads, exports every symbol include/gdr.h declares, and
rejects bad arguments on the host before launching anything (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

import gated_delta_rule_91_b200 as gdr

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "gdr.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDR_API\s+[\w\s\*]*?\b(gdr\w*)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 11
    L = gdr.lib()
    for n in names:
        assert hasattr(L, n), n
        assert n in gdr.SIGNATURES, n


def test_version_and_counter():
    assert gdr.lib().gdr_version() >= 1
    assert gdr.launch_count() >= 0


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first


def _fwd(B=1, T=4, H=1, dk=64, dv=64, dt=gdr.GDR_F32, q=FAKE, k=FAKE, v=FAKE, la=FAKE,
         be=FAKE, S0=None, o=FAKE, ST=None):
    P = ctypes.c_void_p
    return gdr.lib().gdr_fwd(B, T, H, dk, dv, dt, P(q), P(k), P(v), P(la), P(be), P(S0), P(o),
                             P(ST), None, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(T=0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(H=-1), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dk=96), gdr.GDR_ERR_UNSUPPORTED),
    (dict(dv=32), gdr.GDR_ERR_UNSUPPORTED),
    (dict(dt=7), gdr.GDR_ERR_UNSUPPORTED),
    (dict(q=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(o=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(k=FAKE + 4), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(S0=FAKE + 8), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(B=1 << 20, T=1 << 12, H=16), gdr.GDR_ERR_UNSUPPORTED),
])
def test_fwd_rejects_bad_arguments(kw, status):
    assert _fwd(**kw) == status
    assert gdr.lib().gdr_last_error_string().decode().startswith("gdr_fwd")


def test_step_rejects_bad_arguments():
    P = ctypes.c_void_p
    L = gdr.lib()
    assert L.gdr_step(1, 1, 64, 64, gdr.GDR_BF16, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                      None, P(FAKE), None) == gdr.GDR_ERR_INVALID_ARGUMENT
    assert L.gdr_step(1, 1, 48, 64, gdr.GDR_BF16, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                      P(FAKE), P(FAKE), None) == gdr.GDR_ERR_UNSUPPORTED


def test_python_binding_refuses_cpu_tensors():
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises((ValueError, RuntimeError)):
        gdr.gdr_fwd(x, x, x, torch.zeros(1, 4, 1), torch.zeros(1, 4, 1))


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a GPU")
def test_valid_arguments_without_gpu_report_cuda_error():
    # arguments pass validation; the launch then fails cleanly with no device
    assert _fwd() == gdr.GDR_ERR_CUDA


def _prologue(B=1, T=4, H=1, dk=64, dv=64, K=4, dt=gdr.GDR_BF16, x=FAKE, w=FAKE, bias=None,
              st=None, so=None, eps=1e-6, y=FAKE):
    P = ctypes.c_void_p
    return gdr.lib().gdr_block_prologue(B, T, H, dk, dv, K, dt, P(x), P(x), P(x), P(w), P(w), P(w),
                                        P(bias), P(bias), P(bias), P(st), P(so), eps, P(y), P(y),
                                        P(y), None)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(K=0), gdr.GDR_ERR_UNSUPPORTED),
    (dict(K=9), gdr.GDR_ERR_UNSUPPORTED),
    (dict(dk=96), gdr.GDR_ERR_UNSUPPORTED),
    (dict(dt=3), gdr.GDR_ERR_UNSUPPORTED),
    (dict(eps=-1.0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(eps=float("nan")), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(eps=float("inf")), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(x=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(w=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(y=FAKE + 2), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(st=FAKE + 8), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(bias=FAKE + 4), gdr.GDR_ERR_INVALID_ARGUMENT),
])
def test_prologue_rejects_bad_arguments(kw, status):
    assert _prologue(**kw) == status
    assert gdr.lib().gdr_last_error_string().decode().startswith("gdr_block_prologue")


@pytest.mark.parametrize("kw,status", [
    (dict(T=0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dv=256), gdr.GDR_ERR_UNSUPPORTED),
    (dict(eps=-0.5), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(o=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(weight=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(g=FAKE + 8), gdr.GDR_ERR_INVALID_ARGUMENT),
])
def test_epilogue_rejects_bad_arguments(kw, status):
    a = dict(B=1, T=4, H=1, dv=64, dt=gdr.GDR_BF16, o=FAKE, g=None, weight=FAKE, eps=1e-6, y=FAKE)
    a.update(kw)
    P = ctypes.c_void_p
    st = gdr.lib().gdr_block_epilogue(a["B"], a["T"], a["H"], a["dv"], a["dt"], P(a["o"]),
                                      P(a["g"]), P(a["weight"]), a["eps"], P(a["y"]), None)
    assert st == status
    assert gdr.lib().gdr_last_error_string().decode().startswith("gdr_block_epilogue")


@pytest.mark.parametrize("kw,status", [
    (dict(T=0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dv=32), gdr.GDR_ERR_UNSUPPORTED),
    (dict(eps=float("nan")), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dy=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dO=FAKE + 4), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dweight=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(g=FAKE), gdr.GDR_ERR_INVALID_ARGUMENT),            # g without dg
    (dict(dg=FAKE), gdr.GDR_ERR_INVALID_ARGUMENT),           # dg without g
    (dict(ws=None), gdr.GDR_ERR_WORKSPACE),
    (dict(ws_bytes=1024 * 64 * 4 - 1), gdr.GDR_ERR_WORKSPACE),
    (dict(ws=FAKE + 8), gdr.GDR_ERR_INVALID_ARGUMENT),
])
def test_epilogue_bwd_rejects_bad_arguments(kw, status):
    a = dict(B=1, T=4, H=1, dv=64, dt=gdr.GDR_BF16, o=FAKE, g=None, weight=FAKE, eps=1e-6, dy=FAKE,
             dO=FAKE, dg=None, dweight=FAKE, ws=FAKE, ws_bytes=1 << 20)
    a.update(kw)
    P = ctypes.c_void_p
    st = gdr.lib().gdr_block_epilogue_bwd(a["B"], a["T"], a["H"], a["dv"], a["dt"], P(a["o"]), P(a["g"]),
                                          P(a["weight"]), a["eps"], P(a["dy"]), P(a["dO"]), P(a["dg"]),
                                          P(a["dweight"]), P(a["ws"]), a["ws_bytes"], None)
    assert st == status
    assert gdr.lib().gdr_last_error_string().decode().startswith("gdr_block_epilogue_bwd")


def _prologue_bwd(**kw):
    a = dict(B=1, T=4, H=1, dk=64, dv=64, K=4, dt=gdr.GDR_BF16, x=FAKE, w=FAKE, bias=None, st=None,
             eps=1e-6, dy=FAKE, dso=None, dx=FAKE, dw=FAKE, db=None, dsi=None, ws=FAKE, ws_bytes=1 << 24)
    a.update(kw)
    P = ctypes.c_void_p
    return gdr.lib().gdr_block_prologue_bwd(
        a["B"], a["T"], a["H"], a["dk"], a["dv"], a["K"], a["dt"], P(a["x"]), P(a["x"]), P(a["x"]), P(a["w"]),
        P(a["w"]), P(a["w"]), P(a["bias"]), P(a["bias"]), P(a["bias"]), P(a["st"]), a["eps"], P(a["dy"]),
        P(a["dy"]), P(a["dy"]), P(a["dso"]), P(a["dx"]), P(a["dx"]), P(a["dx"]), P(a["dw"]), P(a["dw"]),
        P(a["dw"]), P(a["db"]), P(a["db"]), P(a["db"]), P(a["dsi"]), P(a["ws"]), a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(K=0), gdr.GDR_ERR_UNSUPPORTED),
    (dict(K=9), gdr.GDR_ERR_UNSUPPORTED),
    (dict(dv=32), gdr.GDR_ERR_UNSUPPORTED),
    (dict(eps=-1.0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(x=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dy=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dx=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dw=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(db=FAKE + 4), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dso=FAKE + 2), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dsi=FAKE + 8), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(ws=None), gdr.GDR_ERR_WORKSPACE),
    (dict(ws_bytes=16), gdr.GDR_ERR_WORKSPACE),
])
def test_prologue_bwd_rejects_bad_arguments(kw, status):
    assert _prologue_bwd(**kw) == status
    assert gdr.lib().gdr_last_error_string().decode().startswith("gdr_block_prologue_bwd")


def test_prologue_bwd_workspace_bytes():
    L = gdr.lib()
    # 3H pairs x 32 blocks x max(dk, dv) channels x (taps + bias) fp32
    assert L.gdr_block_prologue_bwd_workspace_bytes(16, 128, 128, 4) == 3 * 16 * 32 * 128 * 5 * 4
    assert L.gdr_block_prologue_bwd_workspace_bytes(2, 64, 128, 6) == 3 * 2 * 32 * 128 * 9 * 4
    assert L.gdr_block_prologue_bwd_workspace_bytes(2, 64, 64, 9) == 0
    assert L.gdr_block_prologue_bwd_workspace_bytes(0, 64, 64, 4) == 0


def test_epilogue_bwd_workspace_bytes():
    assert gdr.lib().gdr_block_epilogue_bwd_workspace_bytes(128) == 1024 * 128 * 4
    assert gdr.lib().gdr_block_epilogue_bwd_workspace_bytes(64) == 1024 * 64 * 4
    assert gdr.lib().gdr_block_epilogue_bwd_workspace_bytes(96) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(R=0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(r=-1), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(r=3), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(S_in=None, S_T=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(M=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dk=32), gdr.GDR_ERR_UNSUPPORTED),
    (dict(S0=FAKE + 4), gdr.GDR_ERR_INVALID_ARGUMENT),
])
def test_seg_combine_rejects_bad_arguments(kw, status):
    a = dict(R=3, r=1, B=1, H=2, dk=64, dv=64, M=FAKE, N=FAKE, S0=None, S_in=FAKE, S_T=None)
    a.update(kw)
    P = ctypes.c_void_p
    st = gdr.lib().gdr_seg_combine(a["R"], a["r"], a["B"], a["H"], a["dk"], a["dv"], P(a["M"]),
                                   P(a["N"]), P(a["S0"]), P(a["S_in"]), P(a["S_T"]), None)
    assert st == status
    assert gdr.lib().gdr_last_error_string().decode().startswith("gdr_seg_combine")


def test_seg_fwd_checks_workspace_and_pointers():
    L, P = gdr.lib(), ctypes.c_void_p
    need = L.gdr_seg_fwd_workspace_bytes(1, 100, 2, 128, 64, gdr.GDR_BF16)
    assert need >= 1 * 100 * 2 * 128 * 2 + 2 * 128 * 128 * 4
    args = [1, 100, 2, 128, 64, gdr.GDR_BF16] + [P(FAKE)] * 9
    assert L.gdr_seg_fwd(*args, P(FAKE), need - 1, None) == gdr.GDR_ERR_WORKSPACE
    assert L.gdr_seg_fwd(*args, None, need, None) == gdr.GDR_ERR_INVALID_ARGUMENT
    bad = [1, 100, 2, 128, 64, gdr.GDR_BF16] + [P(FAKE)] * 7 + [None, P(FAKE)]
    assert L.gdr_seg_fwd(*bad, P(FAKE), need, None) == gdr.GDR_ERR_INVALID_ARGUMENT
    assert L.gdr_seg_fixup(1, 4, 1, 64, 64, gdr.GDR_F32, P(FAKE), None, P(FAKE), None) == \
        gdr.GDR_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(dk=96), gdr.GDR_ERR_UNSUPPORTED),
    (dict(w=None), gdr.GDR_ERR_INVALID_ARGUMENT),
    (dict(S=FAKE + 4), gdr.GDR_ERR_INVALID_ARGUMENT),
])
def test_gdr2_step_rejects_bad_arguments(kw, status):
    a = dict(B=1, H=2, dk=64, dv=64, dt=gdr.GDR_BF16, q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, w=FAKE, S=FAKE,
             o=FAKE)
    a.update(kw)
    P = ctypes.c_void_p
    st = gdr.lib().gdr2_step(a["B"], a["H"], a["dk"], a["dv"], a["dt"], P(a["q"]), P(a["k"]), P(a["v"]),
                             P(a["la"]), P(a["b"]), P(a["w"]), P(a["S"]), P(a["o"]), None)
    assert st == status
    assert gdr.lib().gdr_last_error_string().decode().startswith("gdr2_step")
