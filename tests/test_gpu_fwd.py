"""gdr_fwd on the GPU vs the fp64 oracle, through the C ABI.

Small cases compare every output element and span several chunks and a
ragged tail; the full-size workloads (tiny fp32 B1 H2 T128 d64, and the
layer-shaped bf16 B4 T4096 H16 d128 with random S0) run in the same launch
configuration as the bench and are compared on every head.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_O, TOL_S, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu


def _run(x):
    return gdr.gdr_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]),
                       dev(x["beta"]), dev(x["S0"]))


def _ref(x, bsel=None, hsel=None):
    a = {n: np64(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    if bsel is not None:
        for n in ("q", "k", "v", "log_alpha", "beta"):
            a[n] = np.stack([a[n][b, :, h] for b, h in zip(bsel, hsel)])[:, :, None]
        if a["S0"] is not None:
            a["S0"] = np.stack([a["S0"][b, h] for b, h in zip(bsel, hsel)])[:, None]
    return oracle.gdr_fwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["S0"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 100, 200])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_fwd_small(dtype, T, dk, dv):
    x = synth.gdr_inputs(2, T, 3, dk, dv, dtype, seed=T + dk + dv, s0_std=0.02)
    o, ST = _run(x)
    o_ref, ST_ref = _ref(x)
    assert max_rel(np64(o), o_ref) <= TOL_O[dtype]
    assert fro_rel(np64(ST), ST_ref) <= (TOL_O["f32"] if dtype == "f32" else TOL_S)


def test_fwd_null_state_and_no_final_state():
    x = synth.gdr_inputs(1, 130, 2, 128, 128, "bf16", seed=5)
    assert x["S0"] is None
    o, ST = gdr.gdr_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]),
                        dev(x["beta"]), None, return_state=False)
    assert ST is None
    o_ref, _ = _ref(x)
    assert max_rel(np64(o), o_ref) <= TOL_O["bf16"]


def test_fwd_tiny_f32_workload():
    x = synth.workload_inputs("tiny_f32")
    o, ST = _run(x)
    o_ref, ST_ref = _ref(x)
    assert o.shape == (1, 128, 2, 64) and ST.shape == (1, 2, 64, 64)
    assert max_rel(np64(o), o_ref) <= 1e-4
    assert fro_rel(np64(ST), ST_ref) <= 1e-4


def test_fwd_layer_workload_all_heads():
    """Layer workload B4 T4096 H16 d128 bf16 with random S0, in the bench's
    launch configuration: every output and final state of all 64 heads
    against the oracle (about 2 s of fp64 on 8 host cores)."""
    x = synth.workload_inputs("layer_fwd")
    o, ST = _run(x)
    torch.cuda.synchronize()
    o_ref, ST_ref = _ref(x)
    o_np, ST_np = np64(o), np64(ST)
    assert np.isfinite(o_np).all()
    for b in range(4):
        for h in range(16):
            assert max_rel(o_np[b, :, h], o_ref[b, :, h]) <= TOL_O["bf16"], (b, h)
            assert fro_rel(ST_np[b, h], ST_ref[b, h]) <= TOL_S, (b, h)
    assert max_rel(o_np, o_ref) <= TOL_O["bf16"]


def test_fwd_matches_repeated_steps():
    """The chunkwise forward equals T single-token decode steps (GPU only)."""
    x = synth.gdr_inputs(2, 150, 2, 128, 128, "f32", seed=9, s0_std=0.02)
    o, ST = _run(x)
    S = dev(x["S0"]).clone()
    for t in range(150):
        ot = gdr.gdr_step(dev(x["q"][:, t]), dev(x["k"][:, t]), dev(x["v"][:, t]),
                          dev(x["log_alpha"][:, t]), dev(x["beta"][:, t]), S)
        assert max_rel(np64(ot), np64(o[:, t])) <= 1e-4, t
    assert fro_rel(np64(S), np64(ST)) <= 1e-4


def test_fwd_split_sequence_resume():
    """fwd(0:T) == fwd(0:T1) then fwd(T1:T) started from the state at T1."""
    x = synth.gdr_inputs(1, 300, 4, 128, 128, "bf16", seed=10, s0_std=0.02)
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    o, ST = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    T1 = 100
    cut = lambda n, a, b_: d[n][:, a:b_].contiguous()
    o1, S1 = gdr.gdr_fwd(cut("q", 0, T1), cut("k", 0, T1), cut("v", 0, T1),
                         cut("log_alpha", 0, T1), cut("beta", 0, T1), d["S0"])
    o2, S2 = gdr.gdr_fwd(cut("q", T1, 300), cut("k", T1, 300), cut("v", T1, 300),
                         cut("log_alpha", T1, 300), cut("beta", T1, 300), S1)
    # The two runs place chunk boundaries differently, so the bf16 rounding of
    # the MMA operands (S, U, W: unit roundoff 2^-8) happens at different
    # points: agreement is bounded by the parity tolerances, not by fp32.
    assert max_rel(np64(torch.cat([o1, o2], 1)), np64(o)) <= TOL_O["bf16"]
    assert fro_rel(np64(S2), np64(ST)) <= TOL_S


def test_fwd_deterministic():
    x = synth.gdr_inputs(2, 257, 2, 128, 128, "bf16", seed=11, s0_std=0.02)
    o1, S1 = _run(x)
    o2, S2 = _run(x)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("kernel", ["default", "tc1"])
@pytest.mark.parametrize("T", [64, 129, 1000])
def test_tensor_core_forward_matches_cuda_core_forward(T, kernel, monkeypatch):
    """bf16 d=128 runs on tcgen05 (the two-SM cluster kernel by default, the
    single-CTA kernel with GDR_FWD_KERNEL=tc1); the fp32 CUDA-core kernel on
    the same inputs must agree within the bf16 tolerance (and both with the
    oracle)."""
    x = synth.gdr_inputs(2, T, 3, 128, 128, "bf16", seed=40 + T, s0_std=0.02)
    if kernel != "default":
        monkeypatch.setenv("GDR_FWD_KERNEL", kernel)
    o_tc, S_tc = _run(x)
    gdr.check_status()
    monkeypatch.setenv("GDR_FWD_KERNEL", "simt")
    o_si, S_si = _run(x)
    assert max_rel(np64(o_tc), np64(o_si)) <= TOL_O["bf16"]
    assert fro_rel(np64(S_tc), np64(S_si)) <= TOL_S
    o_ref, S_ref = _ref(x)
    assert max_rel(np64(o_tc), o_ref) <= TOL_O["bf16"]
    assert fro_rel(np64(S_tc), S_ref) <= TOL_S
