"""gdr_bwd on the GPU vs the oracle's hand-derived reverse mode, through the
C ABI.  Tolerances (the pages state none): per gradient tensor
max|d|/max|ref| <= 1e-4 for fp32 inputs and 2e-2 for bf16 inputs; dS0
relative Frobenius <= 1e-2."""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_G, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu

NAMES = ["dq", "dk", "dv", "dlog_alpha", "dbeta"]


def _compare(got, ref, dtype, heads=None):
    for n in NAMES:
        g = np64(got[n])
        if heads is not None:
            g = np.stack([g[b, :, h] for b, h in heads])[:, :, None]
        assert max_rel(g, ref[n]) <= TOL_G[dtype], (n, max_rel(g, ref[n]))
    if got["dS0"] is not None:
        g = np64(got["dS0"])
        if heads is not None:
            g = np.stack([g[b, h] for b, h in heads])[:, None]
        assert fro_rel(g, ref["dS0"]) <= (TOL_G["f32"] if dtype == "f32" else 1e-2)


def _oracle(x, dST, heads=None):
    a = {n: np64(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
    dST = np64(dST)
    if heads is not None:
        for n in ("q", "k", "v", "log_alpha", "beta", "dO"):
            a[n] = np.stack([a[n][b, :, h] for b, h in heads])[:, :, None]
        if a["S0"] is not None:
            a["S0"] = np.stack([a["S0"][b, h] for b, h in heads])[:, None]
        if dST is not None:
            dST = np.stack([dST[b, h] for b, h in heads])[:, None]
    return oracle.gdr_bwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["S0"], a["dO"], dST)


def _gpu(x, dST):
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
    return gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"],
                       dev(dST))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 64, 100, 130])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_bwd_small(dtype, T, dk, dv):
    x = synth.gdr_inputs(2, T, 2, dk, dv, dtype, seed=3 * T + dk, s0_std=0.02, with_dO=True)
    dST = torch.randn(2, 2, dv, dk, generator=torch.Generator().manual_seed(T)) * 0.1
    got = _gpu(x, dST)
    ref = _oracle(x, dST)
    _compare(got, ref, dtype)


def test_bwd_null_state_and_null_dST():
    x = synth.gdr_inputs(1, 90, 3, 128, 128, "f32", seed=21, with_dO=True)
    got = _gpu(x, None)
    ref = _oracle(x, None)
    _compare(got, ref, "f32")


def test_bwd_long_workload_T2048_slice():
    """Long-context workload (B=1, H=16, d=128, bf16, S0=0, dS_T=0), first
    2048 tokens: every gradient of every head against the oracle."""
    x = synth.workload_inputs("long_fwd_bwd")
    xs = {n: (t[:, :2048].contiguous() if t is not None and t.dim() >= 3 and t.shape[1] == 65536
              else t) for n, t in x.items()}
    got = _gpu(xs, None)
    ref = _oracle(xs, None)
    _compare(got, ref, "bf16")


def test_bwd_long_workload_full_length_all_heads():
    """Full T=65536 backward (the timed configuration): every gradient of all
    16 heads against the oracle's reverse mode over the whole sequence
    (about 20 s of fp64 on 8 host cores)."""
    x = synth.workload_inputs("long_fwd_bwd")
    got = _gpu(x, None)
    torch.cuda.synchronize()
    ref = _oracle(x, None)
    _compare(got, ref, "bf16")
    gdr.check_status()


def test_bwd_workspace_is_required():
    x = synth.gdr_inputs(1, 64, 1, 64, 64, "f32", seed=1, with_dO=True)
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "dO")}
    with pytest.raises(gdr.GdrError) as e:
        gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, d["dO"],
                    workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == gdr.GDR_ERR_WORKSPACE


def test_bwd_deterministic():
    x = synth.gdr_inputs(1, 200, 2, 128, 128, "bf16", seed=4, s0_std=0.02, with_dO=True)
    a = _gpu(x, None)
    b = _gpu(x, None)
    for n in NAMES + ["dS0"]:
        assert torch.equal(a[n], b[n]), n


@pytest.mark.parametrize("T", [64, 129, 1000])
def test_tensor_core_backward_matches_cuda_core_backward(T, monkeypatch):
    """bf16 d=128 runs on tcgen05 (recompute, dS pass, chunk-parallel
    gradients); the fp32 CUDA-core backward (GDR_BWD_KERNEL=simt) on the same
    inputs must agree within the bf16 tolerance, and both with the oracle."""
    x = synth.gdr_inputs(2, T, 3, 128, 128, "bf16", seed=60 + T, s0_std=0.02, with_dO=True)
    dST = torch.randn(2, 3, 128, 128, generator=torch.Generator().manual_seed(T)) * 0.05
    got = _gpu(x, dST)
    gdr.check_status()
    monkeypatch.setenv("GDR_BWD_KERNEL", "simt")
    ref_si = _gpu(x, dST)
    for n in NAMES:
        assert max_rel(np64(got[n]), np64(ref_si[n])) <= TOL_G["bf16"], n
    assert fro_rel(np64(got["dS0"]), np64(ref_si["dS0"])) <= 1e-2
    _compare(got, _oracle(x, dST), "bf16")
