"""gdr_bwd_noalloc: the backward for callers that cannot allocate device
memory (a memory pool or arena that owns the whole device, a runtime that
forbids cudaMalloc once started, an allocation-free hot loop).  It takes the
same inputs and outputs as gdr_bwd but no workspace: its scratch is a fixed
64 MiB array inside libgdr.so.

Checked through the C ABI: two consecutive calls (different inputs, the
second reusing the scratch the first left behind) must match gdr_bwd with a
caller workspace and the oracle's reverse mode within the gradient
tolerances the other tests use; a warmed-up call must leave the device's
free memory and torch's allocation count unchanged; and a problem whose
scratch does not fit is refused on the host.  This file sorts last so that
a run stopping at its first failure has run everything else.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_G, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def _noalloc(d, dtype_code, dST):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    out = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]),
               dv=torch.empty_like(d["v"]), dlog_alpha=torch.empty_like(d["log_alpha"]),
               dbeta=torch.empty_like(d["beta"]),
               dS0=torch.empty(B, H, dv, dk, dtype=torch.float32, device="cuda"))
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = gdr.lib().gdr_bwd_noalloc(B, T, H, dk, dv, dtype_code, P(d["q"]), P(d["k"]), P(d["v"]),
                                   P(d["log_alpha"]), P(d["beta"]), P(d["S0"]), P(d["dO"]),
                                   P(dST), P(out["dq"]), P(out["dk"]), P(out["dv"]),
                                   P(out["dlog_alpha"]), P(out["dbeta"]), P(out["dS0"]), stream)
    gdr.check(st)
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_backward_matches_workspace_backward_twice(dtype):
    code = gdr.GDR_F32 if dtype == "f32" else gdr.GDR_BF16
    for call, (T, seed) in enumerate([(300, 71), (130, 72)]):
        x = synth.gdr_inputs(1, T, 3, 128, 128, dtype, seed=seed, s0_std=0.02, with_dO=True)
        d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
        dST = dev(torch.randn(1, 3, 128, 128, generator=torch.Generator().manual_seed(seed)) * 0.1)
        got = _noalloc(d, code, dST)
        ref = gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"], dST)
        torch.cuda.synchronize()
        for n in NAMES[:-1]:
            assert max_rel(np64(got[n]), np64(ref[n])) <= TOL_G[dtype], (call, n)
        assert fro_rel(np64(got["dS0"]), np64(ref["dS0"])) <= TOL_G[dtype], call
        a = {n: np64(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
        orc = oracle.gdr_bwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["S0"], a["dO"],
                             np64(dST))
        for n in NAMES[:-1]:
            assert max_rel(np64(got[n]), orc[n]) <= TOL_G[dtype], (call, n, "oracle")
        assert fro_rel(np64(got["dS0"]), orc["dS0"]) <= (TOL_G["f32"] if dtype == "f32" else 1e-2), call


def test_noalloc_backward_allocates_no_device_memory():
    """After a first call (which resolves the scratch array's address), a call
    changes neither the device's free memory nor torch's allocation count."""
    x = synth.gdr_inputs(1, 200, 2, 128, 128, "bf16", seed=73, s0_std=0.02, with_dO=True)
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
    B, T, H, dk = d["q"].shape
    out = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]),
               dv=torch.empty_like(d["v"]), dlog_alpha=torch.empty_like(d["log_alpha"]),
               dbeta=torch.empty_like(d["beta"]),
               dS0=torch.empty(B, H, 128, dk, dtype=torch.float32, device="cuda"))
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        gdr.check(gdr.lib().gdr_bwd_noalloc(
            B, T, H, dk, 128, gdr.GDR_BF16, P(d["q"]), P(d["k"]), P(d["v"]), P(d["log_alpha"]),
            P(d["beta"]), P(d["S0"]), P(d["dO"]), None, P(out["dq"]), P(out["dk"]), P(out["dv"]),
            P(out["dlog_alpha"]), P(out["dbeta"]), P(out["dS0"]), stream))

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_noalloc_refuses_a_problem_larger_than_its_scratch():
    need = gdr.lib().gdr_bwd_workspace_bytes(1, 65536, 16, 128, 128, gdr.GDR_BF16)
    assert need > (64 << 20)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: refused before any launch
    st = gdr.lib().gdr_bwd_noalloc(1, 65536, 16, 128, 128, gdr.GDR_BF16, fake, fake, fake, fake,
                                   fake, None, fake, None, fake, fake, fake, fake, fake, None,
                                   None)
    assert st == gdr.GDR_ERR_WORKSPACE
    assert "static scratch" in gdr.lib().gdr_last_error_string().decode()
