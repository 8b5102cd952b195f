"""GPU parity of gdr2_step (Gated DeltaNet-2 decode, state in place) against
the fp64 oracle's Gated Delta Rule-2 forward run one token at a time, and
against the GPU forward over the same tokens."""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_O, TOL_S, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu


def _tok(x, n, t):
    return x[n][:, t].contiguous().cuda()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_decode_chain_matches_oracle(dtype, dk, dv):
    steps = 5
    x = synth.gdr2_inputs(3, steps, 2, dk, dv, dtype, seed=dk + dv, s0_std=0.02, b_max=2.0)
    S = x["S0"].clone().cuda()
    S_ref = np64(x["S0"])
    for t in range(steps):
        o = gdr.gdr2_step(*(_tok(x, n, t) for n in ("q", "k", "v", "log_alpha", "b", "w")), S)
        sl = lambda n: np64(x[n][:, t:t + 1])
        o_ref, S_ref = oracle.gdr2_fwd(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("b"), sl("w"), S_ref)
        assert max_rel(np64(o), o_ref[:, 0]) <= TOL_O[dtype], t
    gdr.check_status()
    assert fro_rel(np64(S), S_ref) <= (TOL_S if dtype == "bf16" else 1e-4)


def test_decode_chain_equals_forward_on_gpu():
    T = 100
    x = synth.gdr2_inputs(2, T, 4, 128, 128, "bf16", seed=3, s0_std=0.02)
    d = {n: x[n].cuda() for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}
    o_f, S_f = gdr.gdr2_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    S = d["S0"].clone()
    outs = [gdr.gdr2_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")), S)
            for t in range(T)]
    gdr.check_status()
    assert max_rel(np64(torch.stack(outs, dim=1)), np64(o_f)) <= TOL_O["bf16"]
    assert fro_rel(np64(S), np64(S_f)) <= TOL_S


def test_decode_workload_sampled_heads():
    B, H, d = 256, 16, 128
    x = synth.gdr2_inputs(B, 2, H, d, d, "bf16", seed=11, s0_std=0.02)
    S = x["S0"].clone().cuda()
    outs = [gdr.gdr2_step(*(_tok(x, n, t) for n in ("q", "k", "v", "log_alpha", "b", "w")), S) for t in range(2)]
    gdr.check_status()
    for b, h in ((0, 0), (100, 7), (255, 15)):
        sl = lambda n: np64(x[n][b:b + 1, :, h:h + 1])
        o_ref, S_ref = oracle.gdr2_fwd(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("b"), sl("w"),
                                       np64(x["S0"][b:b + 1, h:h + 1]))
        for t in range(2):
            assert max_rel(np64(outs[t][b:b + 1, h:h + 1]), o_ref[:, t]) <= TOL_O["bf16"]
        assert fro_rel(np64(S[b:b + 1, h:h + 1]), S_ref) <= TOL_S
