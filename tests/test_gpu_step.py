"""gdr_step (single-token decode) on the GPU vs the fp64 oracle, through the
C ABI.  Tolerances: max|d o|/max|o_ref| <= 1e-4 (fp32 inputs) or 2e-2 (bf16),
state relative Frobenius <= 1e-2."""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_O, TOL_S, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_step_sequence_small(dtype, dk, dv):
    B, H, steps, seed = 3, 2, 40, 17
    S = synth.decode_state(B, H, dk, dv, seed)
    S_dev = dev(S)
    S_ref = np64(S)
    for t in range(steps):
        x = synth.decode_step_inputs(B, H, dk, dv, dtype, seed, t)
        o = gdr.gdr_step(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]),
                         dev(x["beta"]), S_dev)
        o_ref, S_ref = oracle.gdr_step(np64(x["q"]), np64(x["k"]), np64(x["v"]),
                                       np64(x["log_alpha"]), np64(x["beta"]), S_ref)
        assert max_rel(np64(o), o_ref) <= TOL_O[dtype], t
    assert fro_rel(np64(S_dev), S_ref) <= (1e-5 if dtype == "f32" else TOL_S)


def test_decode_workload_all_heads():
    """Decode workload B=256 H=16 d=128, bf16, 1024 consecutive steps on the
    full state: o of all 4096 heads at every step and the whole state after
    the last step against the oracle, which follows the full fp64 state in
    place (about 45 ms per step on 8 host cores)."""
    w = synth.WORKLOADS["decode"]
    B, H, dk, dv = w.B, w.H, w.dk, w.dv
    S = synth.decode_state(B, H, dk, dv, w.seed)
    S_dev = dev(S)
    S_ref = np.ascontiguousarray(np64(S))
    worst = 0.0
    for t in range(w.steps):
        x = synth.decode_step_inputs(B, H, dk, dv, w.dtype, w.seed, t)
        o = gdr.gdr_step(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]),
                         dev(x["beta"]), S_dev)
        o_ref = oracle.gdr_step_inplace(np64(x["q"]), np64(x["k"]), np64(x["v"]),
                                        np64(x["log_alpha"]), np64(x["beta"]), S_ref)
        err = max_rel(np64(o), o_ref)
        worst = max(worst, err)
        assert err <= TOL_O["bf16"], (t, err)
    torch.cuda.synchronize()
    assert fro_rel(np64(S_dev), S_ref) <= TOL_S
    gdr.check_status()


def test_step_rejects_timeout_free():
    """The decode kernel has no waits; the status word stays clear."""
    gdr.check_status()
