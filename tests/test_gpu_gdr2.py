"""gdr2_fwd (Gated DeltaNet-2) on the GPU vs the fp64 oracle, through the
C ABI, plus the collapse to the scalar-gate rule on the GPU."""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_O, TOL_S, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu


def _gpu(x):
    return gdr.gdr2_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]),
                        dev(x["b"]), dev(x["w"]), dev(x["S0"]))


def _oracle(x, heads=None):
    a = {n: np64(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}
    if heads is not None:
        for n in ("q", "k", "v", "log_alpha", "b", "w"):
            a[n] = np.stack([a[n][b, :, h] for b, h in heads])[:, :, None]
        if a["S0"] is not None:
            a["S0"] = np.stack([a["S0"][b, h] for b, h in heads])[:, None]
    return oracle.gdr2_fwd(a["q"], a["k"], a["v"], a["log_alpha"], a["b"], a["w"], a["S0"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 64, 100, 130])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_gdr2_small(dtype, T, dk, dv):
    x = synth.gdr2_inputs(2, T, 2, dk, dv, dtype, seed=T + 7 * dk + dv, s0_std=0.02)
    o, ST = _gpu(x)
    o_ref, ST_ref = _oracle(x)
    assert max_rel(np64(o), o_ref) <= TOL_O[dtype]
    assert fro_rel(np64(ST), ST_ref) <= (TOL_O["f32"] if dtype == "f32" else TOL_S)


def test_gdr2_workload_all_heads():
    """Gated DeltaNet-2 workload B4 T4096 H16 d128 bf16: every head's outputs
    and final state against the oracle."""
    x = synth.workload_inputs("gdn2_fwd")
    o, ST = _gpu(x)
    torch.cuda.synchronize()
    o_ref, ST_ref = _oracle(x)
    o_np, ST_np = np64(o), np64(ST)
    assert np.isfinite(o_np).all()
    for b in range(4):
        for h in range(16):
            assert max_rel(o_np[b, :, h], o_ref[b, :, h]) <= TOL_O["bf16"], (b, h)
            assert fro_rel(ST_np[b, h], ST_ref[b, h]) <= TOL_S, (b, h)


def test_gdr2_collapses_to_gated_delta_rule_on_gpu():
    """b = w = beta*1 and a scalar decay broadcast to every channel give the
    scalar-gate rule's outputs (Gated DeltaNet-2 page: both gates one
    scalar and the decay a scalar -> Gated DeltaNet)."""
    x = synth.gdr_inputs(2, 150, 3, 128, 128, "f32", seed=31, s0_std=0.02)
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    o1, S1 = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    la = d["log_alpha"][..., None].expand(-1, -1, -1, 128).contiguous()
    bw = d["beta"][..., None].expand(-1, -1, -1, 128).contiguous()
    o2, S2 = gdr.gdr2_fwd(d["q"], d["k"], d["v"], la, bw, bw, d["S0"])
    assert max_rel(np64(o2), np64(o1)) <= 1e-4
    assert fro_rel(np64(S2), np64(S1)) <= 1e-4


@pytest.mark.parametrize("kernel", ["default", "tc1"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 300])
def test_gdr2_cluster_and_single_cta_kernels(kernel, T, monkeypatch):
    """The default two-SM cluster kernel and the single-CTA tensor-core kernel
    (GDR2_FWD_KERNEL=tc1) against the oracle: one token, a chunk less one, a
    whole chunk, one past it, and ragged multi-chunk lengths."""
    if kernel != "default":
        monkeypatch.setenv("GDR2_FWD_KERNEL", kernel)
    x = synth.gdr2_inputs(2, T, 3, 128, 128, "bf16", seed=400 + T, s0_std=0.02)
    o, S = _gpu(x)
    gdr.check_status()
    o_ref, S_ref = _oracle(x)
    assert max_rel(np64(o), o_ref) <= TOL_O["bf16"]
    assert fro_rel(np64(S), S_ref) <= TOL_S


@pytest.mark.parametrize("kernel", ["default", "tc1"])
def test_gdr2_exact_chunks_between_ordinary_ones(kernel, monkeypatch):
    """A decay spike (log alpha = -100 in four channels at one token) puts
    chunks 1 and 3 past e^80: they take the exact path, the chunks around
    them the tensor-core form, and the state must carry across both kinds.
    T = 300 ends on a ragged chunk."""
    if kernel != "default":
        monkeypatch.setenv("GDR2_FWD_KERNEL", kernel)
    x = synth.gdr2_inputs(2, 300, 2, 128, 128, "bf16", seed=88, s0_std=0.02)
    la = x["log_alpha"].clone()
    la[:, 70, :, 8:12] = -100.0
    la[:, 200, :, 100:104] = -100.0
    x["log_alpha"] = la
    o, S = _gpu(x)
    gdr.check_status()
    o_ref, S_ref = _oracle(x)
    assert max_rel(np64(o), o_ref) <= TOL_O["bf16"]
    assert fro_rel(np64(S), S_ref) <= TOL_S


@pytest.mark.parametrize("T", [64, 129, 1000])
def test_tensor_core_gdr2_matches_cuda_core_gdr2(T, monkeypatch):
    """bf16 d=128 runs on tcgen05; the fp32 CUDA-core kernel
    (GDR2_FWD_KERNEL=simt) on the same inputs must agree within the bf16
    tolerance, and both with the oracle."""
    x = synth.gdr2_inputs(2, T, 3, 128, 128, "bf16", seed=90 + T, s0_std=0.02)
    o_tc, S_tc = _gpu(x)
    gdr.check_status()
    monkeypatch.setenv("GDR2_FWD_KERNEL", "simt")
    o_si, S_si = _gpu(x)
    assert max_rel(np64(o_tc), np64(o_si)) <= TOL_O["bf16"]
    assert fro_rel(np64(S_tc), np64(S_si)) <= TOL_S
    o_ref, S_ref = _oracle(x)
    assert max_rel(np64(o_tc), o_ref) <= TOL_O["bf16"]
    assert fro_rel(np64(S_tc), S_ref) <= TOL_S


@pytest.mark.parametrize("kernel", ["default", "tc1"])
def test_gdr2_strong_decay_takes_the_exact_path(kernel, monkeypatch):
    """Channels that decay by e^-3 per token fall by e^-192 over a chunk, past
    what K/E can hold in a bf16 operand; those chunks evaluate A and P term
    by term.  Half the heads decay strongly in half the channels; all must
    still match the oracle, on the two-SM kernel and the single-CTA one."""
    if kernel != "default":
        monkeypatch.setenv("GDR2_FWD_KERNEL", kernel)
    x = synth.gdr2_inputs(1, 200, 4, 128, 128, "bf16", seed=77, s0_std=0.02)
    la = x["log_alpha"].clone()
    la[:, :, :2, :64] = -3.0
    x["log_alpha"] = la
    o, S = _gpu(x)
    gdr.check_status()
    o_ref, S_ref = _oracle(x)
    assert max_rel(np64(o), o_ref) <= TOL_O["bf16"]
    assert fro_rel(np64(S), S_ref) <= TOL_S


def test_gdr2_deterministic():
    x = synth.gdr2_inputs(2, 300, 3, 128, 128, "bf16", seed=55, s0_std=0.02)
    o1, S1 = _gpu(x)
    o2, S2 = _gpu(x)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_gdr2_split_sequence_resume():
    """Running [0, t) then [t, T) from the first part's final state gives the
    same outputs and state as one pass (the state is the whole carry)."""
    x = synth.gdr2_inputs(1, 700, 2, 128, 128, "bf16", seed=56, s0_std=0.02)
    o, S = _gpu(x)
    t = 320  # a chunk boundary; the second part starts a fresh chunk grid
    a = {n: (v[:, :t].contiguous() if v is not None and v.dim() == 4 and v.shape[1] == 700 else v)
         for n, v in x.items()}
    b = {n: (v[:, t:].contiguous() if v is not None and v.dim() == 4 and v.shape[1] == 700 else v)
         for n, v in x.items()}
    oa, Sa = _gpu(a)
    b["S0"] = Sa.cpu()
    ob, Sb = _gpu(b)
    o2 = torch.cat([oa, ob], dim=1)
    assert max_rel(np64(o2), np64(o)) <= TOL_O["bf16"]
    assert fro_rel(np64(Sb), np64(S)) <= TOL_S


def test_gdr2_null_state_and_no_final_state():
    x = synth.gdr2_inputs(1, 150, 2, 128, 128, "bf16", seed=57)
    assert x["S0"] is None
    o, S = gdr.gdr2_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["b"]),
                        dev(x["w"]), None, return_state=False)
    assert S is None
    o_ref, _ = _oracle(x)
    assert max_rel(np64(o), o_ref) <= TOL_O["bf16"]


@pytest.mark.parametrize("kernel", ["default", "tc1", "simt"])
def test_gdr2_negative_eigenvalue_erase_gate(kernel, monkeypatch):
    """Erase gate b in (0, 2) (the negative-eigenvalue range): the erase
    factor's eigenvalue along k reaches -1, and over 1000 tokens both
    kernels must still match the oracle."""
    if kernel != "default":
        monkeypatch.setenv("GDR2_FWD_KERNEL", kernel)
    x = synth.gdr2_inputs(2, 1000, 2, 128, 128, "bf16", seed=58, s0_std=0.02, b_max=2.0)
    assert float(x["b"].max()) > 1.5
    o, S = _gpu(x)
    gdr.check_status()
    o_ref, S_ref = _oracle(x)
    assert max_rel(np64(o), o_ref) <= TOL_O["bf16"]
    assert fro_rel(np64(S), S_ref) <= TOL_S
