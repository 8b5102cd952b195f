"""gdr2_bwd (Gated DeltaNet-2 backward) on the GPU vs the oracle's reverse
mode, through the C ABI.  Tolerances as for gdr_bwd: per gradient tensor
max|d|/max|ref| <= 1e-4 for fp32 inputs and 2e-2 for bf16 inputs; dS0
relative Frobenius <= 1e-2 (bf16) / 1e-4 (fp32)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_G, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu

NAMES = ["dq", "dk", "dv", "dlog_alpha", "db", "dw"]


def _inputs(B, T, H, dk, dv, dtype, seed, b_max=1.0):
    x = synth.gdr2_inputs(B, T, H, dk, dv, dtype, seed=seed, s0_std=0.02, b_max=b_max)
    g = torch.Generator().manual_seed(seed + 1)
    x["dO"] = torch.randn(B, T, H, dv, generator=g).to(x["q"].dtype)
    return x


def _gpu(x, dST):
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0", "dO")}
    return gdr.gdr2_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], d["dO"], dev(dST))


def _oracle(x, dST, heads=None):
    a = {n: np64(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0", "dO")}
    dST = np64(dST)
    if heads is not None:
        for n in ("q", "k", "v", "log_alpha", "b", "w", "dO"):
            a[n] = np.stack([a[n][b, :, h] for b, h in heads])[:, :, None]
        a["S0"] = np.stack([a["S0"][b, h] for b, h in heads])[:, None]
        if dST is not None:
            dST = np.stack([dST[b, h] for b, h in heads])[:, None]
    return oracle.gdr2_bwd(a["q"], a["k"], a["v"], a["log_alpha"], a["b"], a["w"], a["S0"], a["dO"], dST)


def _compare(got, ref, dtype, heads=None):
    for n in NAMES:
        g = np64(got[n])
        if heads is not None:
            g = np.stack([g[b, :, h] for b, h in heads])[:, :, None]
        assert max_rel(g, ref[n]) <= TOL_G[dtype], (n, max_rel(g, ref[n]))
    g = np64(got["dS0"])
    if heads is not None:
        g = np.stack([g[b, h] for b, h in heads])[:, None]
    assert fro_rel(g, ref["dS0"]) <= (TOL_G["f32"] if dtype == "f32" else 1e-2)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 64, 100, 130])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_gdr2_bwd_small(dtype, T, dk, dv):
    x = _inputs(2, T, 2, dk, dv, dtype, seed=5 * T + dk + dv)
    dST = torch.randn(2, 2, dv, dk, generator=torch.Generator().manual_seed(T)) * 0.1
    got = _gpu(x, dST)
    gdr.check_status()
    _compare(got, _oracle(x, dST), dtype)


def test_gdr2_bwd_workload_sampled_heads():
    """The Gated DeltaNet-2 workload shape (B4 T4096 H16 d128 bf16): two heads
    against the oracle over the whole sequence."""
    x = _inputs(4, 4096, 16, 128, 128, "bf16", seed=4)
    got = _gpu(x, None)
    torch.cuda.synchronize()
    gdr.check_status()
    heads = [(0, 3), (3, 12)]
    _compare(got, _oracle(x, None, heads), "bf16", heads)


def test_gdr2_bwd_deterministic():
    x = _inputs(1, 200, 2, 128, 128, "bf16", seed=9)
    a = _gpu(x, None)
    b = _gpu(x, None)
    for n in NAMES + ["dS0"]:
        assert torch.equal(a[n], b[n]), n


def test_gdr2_bwd_collapses_to_gdr_bwd_on_gpu():
    """b = w = beta*1 and a scalar decay broadcast to every channel: the
    Gated DeltaNet-2 gradients reduce to the scalar-gate rule's (dlog alpha
    summed over channels, dbeta = sum db + sum dw), across the two GPU
    backward paths."""
    x = synth.gdr_inputs(2, 150, 2, 128, 128, "f32", seed=33, s0_std=0.02, with_dO=True)
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
    g1 = gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"])
    la = d["log_alpha"][..., None].expand(-1, -1, -1, 128).contiguous()
    bw = d["beta"][..., None].expand(-1, -1, -1, 128).contiguous()
    g2 = gdr.gdr2_bwd(d["q"], d["k"], d["v"], la, bw, bw, d["S0"], d["dO"])
    for n in ("dq", "dk", "dv", "dS0"):
        assert max_rel(np64(g2[n]), np64(g1[n])) <= 1e-4, n
    assert max_rel(np64(g2["dlog_alpha"].sum(-1)), np64(g1["dlog_alpha"])) <= 1e-4
    assert max_rel(np64(g2["db"].sum(-1) + g2["dw"].sum(-1)), np64(g1["dbeta"])) <= 1e-4


@pytest.mark.parametrize("dtype,dk,dv", [("f32", 64, 64), ("f32", 128, 128), ("bf16", 128, 128),
                                          ("bf16", 64, 128)])
def test_gdr2_bwd_strong_decay(dtype, dk, dv):
    """Chunks in which some channel decays by more than e^80 (log alpha = -3
    on 8 of the key channels: e^-192 over 64 tokens) go through the exact
    token-by-token reverse; the others through the chunk form.  T = 229 mixes
    both (the decay is applied from token 70 on) and ends in a ragged chunk."""
    x = _inputs(2, 229, 2, dk, dv, dtype, seed=10 + dk + dv)
    x["log_alpha"][:, 70:, :, :8] = -3.0
    dST = torch.randn(2, 2, dv, dk, generator=torch.Generator().manual_seed(12)) * 0.1
    got = _gpu(x, dST)
    gdr.check_status()
    _compare(got, _oracle(x, dST), dtype)


@pytest.mark.parametrize("la", [-0.3, -0.35])
def test_gdr2_bwd_decay_near_the_tensor_core_span(la):
    """A full chunk decays by e^-19.2 (log alpha = -0.3: products on the
    tensor cores) or e^-22.4 (-0.35: products in fp32 in the reverse pass) on
    every channel; both must match the oracle."""
    x = _inputs(1, 200, 2, 128, 128, "bf16", seed=81)
    x["log_alpha"][:] = la
    dST = torch.randn(1, 2, 128, 128, generator=torch.Generator().manual_seed(13)) * 0.1
    got = _gpu(x, dST)
    gdr.check_status()
    _compare(got, _oracle(x, dST), "bf16")


def test_gdr2_bwd_strong_decay_every_channel():
    """Every channel decays past e^80 in every chunk (log alpha = -2): the
    whole sequence takes the exact path, with the erase gate in (0, 2)."""
    x = _inputs(1, 150, 2, 128, 128, "bf16", seed=77, b_max=2.0)
    x["log_alpha"][:] = -2.0
    got = _gpu(x, None)
    gdr.check_status()
    _compare(got, _oracle(x, None), "bf16")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gdr2_bwd_negative_eigenvalue_erase_gate(dtype):
    # b in (0, 2): the erase factor can reflect; the gradients must still
    # match the oracle's reverse mode
    x = _inputs(2, 200, 2, 128, 128, dtype, seed=41, b_max=2.0)
    assert float(x["b"].max()) > 1.0
    dST = torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(3)) * 0.1
    got = _gpu(x, dST)
    gdr.check_status()
    _compare(got, _oracle(x, dST), dtype)
