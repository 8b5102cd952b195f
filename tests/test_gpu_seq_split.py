"""GPU parity of the sequence split (gdr_seg_fwd -> exchange -> gdr_seg_combine
-> gdr_seg_fixup) against the fp64 oracle over the whole sequence.  The R
ranks are emulated on one GPU: each segment's calls run in turn and the
exchange is a stack of the segments' (M, N); no kernel waits on another."""
import os
import socket

import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_O, TOL_S, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu


def emulate(x, cuts, S0):
    """Run the split over segments [cuts[i], cuts[i+1]) on one GPU."""
    parts = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        parts.append(gdr.gdr_seg_fwd(*(x[n][:, a:b].clone() for n in ("q", "k", "v", "log_alpha", "beta"))))
    M_all = torch.stack([p[3] for p in parts])
    N_all = torch.stack([p[2] for p in parts])
    outs, S_T = [], None
    for r, (o0, qt, _, _) in enumerate(parts):
        S_in, S_T = gdr.gdr_seg_combine(M_all, N_all, r, S0)
        outs.append(gdr.gdr_seg_fixup(qt, S_in, o0))
    gdr.check_status()
    return torch.cat(outs, dim=1), S_T


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 64), ("f32", 128, 64)])
@pytest.mark.parametrize("cuts", [[], [500], [130, 640], [1, 300, 301]])
def test_split_matches_oracle(dtype, dk, dv, cuts):
    T = 1000
    x = synth.gdr_inputs(1, T, 2, dk, dv, dtype, seed=len(cuts) + dk, s0_std=0.02)
    d = {n: dev(t) for n, t in x.items() if t is not None}
    o, S_T = emulate(d, [0] + cuts + [T], d["S0"])
    o_ref, S_ref = oracle.gdr_fwd(np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["log_alpha"]),
                                  np64(x["beta"]), np64(x["S0"]))
    assert max_rel(np64(o), o_ref) <= TOL_O[dtype]
    assert fro_rel(np64(S_T), S_ref) <= (TOL_S if dtype == "bf16" else 1e-4)


def test_split_agrees_with_one_pass_on_gpu():
    T = 2048
    x = synth.gdr_inputs(2, T, 4, 128, 128, "bf16", seed=9, s0_std=0.02)
    d = {n: dev(t) for n, t in x.items() if t is not None}
    o1, S1 = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    o, S_T = emulate(d, [0, 512, 1024, 1536, 2048], d["S0"])
    assert max_rel(np64(o), np64(o1)) <= TOL_O["bf16"]
    assert fro_rel(np64(S_T), np64(S1)) <= TOL_S


def test_combine_kernel_matches_numpy():
    rng = np.random.default_rng(0)
    R, B, H, dk, dv = 5, 2, 3, 128, 64
    M = (rng.standard_normal((R, B, H, dk, dk)) * 0.08).astype(np.float32)
    N = rng.standard_normal((R, B, H, dv, dk)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dv, dk)).astype(np.float32)
    for r in range(R):
        S_in, S_T = gdr.gdr_seg_combine(torch.from_numpy(M).cuda(), torch.from_numpy(N).cuda(), r,
                                        torch.from_numpy(S0).cuda())
        S = S0.astype(np.float64)
        ref_in = None
        for j in range(R):
            if j == r:
                ref_in = S.copy()
            S = S @ M[j].astype(np.float64) + N[j]
        assert fro_rel(np64(S_in), ref_in) <= 1e-5
        assert fro_rel(np64(S_T), S) <= 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fixup_kernel_matches_numpy(dtype):
    rng = np.random.default_rng(1)
    B, T, H, dk, dv = 2, 77, 3, 64, 128
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    qt = torch.from_numpy(rng.standard_normal((B, T, H, dk)).astype(np.float32)).to(tdt).cuda()
    o = torch.from_numpy(rng.standard_normal((B, T, H, dv)).astype(np.float32)).to(tdt).cuda()
    S = torch.from_numpy(rng.standard_normal((B, H, dv, dk)).astype(np.float32) * 0.1).cuda()
    ref = np64(o) + np.einsum("bhij,bthj->bthi", np64(S), np64(qt))
    gdr.gdr_seg_fixup(qt, S, o)
    torch.cuda.synchronize()
    assert max_rel(np64(o), ref) <= (1e-5 if dtype == "f32" else 8e-3)


def test_long_sequence_split_in_eight_sampled_heads():
    # B1 T65536 H16 d128 bf16 split into 8 segments of 8192 tokens; the
    # oracle follows two heads over the whole sequence
    x = synth.workload_inputs("long_fwd_bwd")
    d = {n: dev(t) for n, t in x.items() if t is not None and n != "dO"}
    T = d["q"].shape[1]
    S0 = d.get("S0")
    o, S_T = emulate(d, [i * T // 8 for i in range(9)], S0)
    for h in (3, 12):
        sl = lambda n: np64(x[n][:, :, h:h + 1])
        s0 = None if x.get("S0") is None else np64(x["S0"][:, h:h + 1])
        o_ref, S_ref = oracle.gdr_fwd(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("beta"), s0)
        assert max_rel(np64(o[:, :, h:h + 1]), o_ref) <= TOL_O["bf16"]
        assert fro_rel(np64(S_T[:, h:h + 1]), S_ref) <= TOL_S


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_orchestrator_over_one_rank_nccl_group():
    # the product path end to end (NCCL all-gather included) with one rank
    import torch.distributed as dist
    from gated_delta_rule_91_b200.seq_split import seq_split_fwd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
    try:
        x = synth.gdr_inputs(1, 300, 2, 128, 128, "bf16", seed=2, s0_std=0.02)
        d = {n: dev(t) for n, t in x.items() if t is not None}
        o, S_T = seq_split_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
        o1, S1 = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
        torch.cuda.synchronize()
        assert max_rel(np64(o), np64(o1)) <= TOL_O["bf16"]
        assert fro_rel(np64(S_T), np64(S1)) <= TOL_S
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T", [1, 100, 128, 1000])
def test_tensor_core_fixup_matches_cuda_core_fixup(T, monkeypatch):
    rng = np.random.default_rng(T)
    B, H = 2, 3
    qt = torch.from_numpy(rng.standard_normal((B, T, H, 128)).astype(np.float32)).to(torch.bfloat16).cuda()
    o = torch.from_numpy(rng.standard_normal((B, T, H, 128)).astype(np.float32)).to(torch.bfloat16).cuda()
    S = torch.from_numpy(rng.standard_normal((B, H, 128, 128)).astype(np.float32) * 0.1).cuda()
    ref = np64(o) + np.einsum("bhij,bthj->bthi", np64(S), np64(qt))
    o_tc = gdr.gdr_seg_fixup(qt, S, o.clone())
    monkeypatch.setenv("GDR_SEG_FIXUP", "simt")
    o_simt = gdr.gdr_seg_fixup(qt, S, o.clone())
    gdr.check_status()
    # the tensor-core product rounds S_in to bf16 (relative 2^-9 per term)
    assert max_rel(np64(o_tc), ref) <= 1e-2
    assert max_rel(np64(o_simt), ref) <= 8e-3


@pytest.mark.parametrize("B,T,H,R", [(1, 16384, 16, 2), (1, 8192, 8, 4), (2, 8192, 4, 4)])
def test_gdr_fwd_runs_long_sequences_as_parallel_segments(B, T, H, R, monkeypatch):
    # few (b, h) and a long T: gdr_fwd asks for a workspace and runs R
    # segments of the sequence in parallel on this GPU; it must agree with the
    # unsplit kernel and with the oracle
    L = gdr.lib()
    assert L.gdr_fwd_workspace_bytes(B, T, H, 128, 128, gdr.GDR_BF16) > 0
    x = synth.gdr_inputs(B, T, H, 128, 128, "bf16", seed=R + B, s0_std=0.02)
    d = {n: dev(t) for n, t in x.items() if t is not None}
    o, S_T = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    monkeypatch.setenv("GDR_FWD_SPLIT", "off")
    assert L.gdr_fwd_workspace_bytes(B, T, H, 128, 128, gdr.GDR_BF16) == 0
    o1, S1 = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    gdr.check_status()
    assert max_rel(np64(o), np64(o1)) <= TOL_O["bf16"]
    assert fro_rel(np64(S_T), np64(S1)) <= TOL_S
    h = H - 1
    sl = lambda n: np64(x[n][:, :, h:h + 1])
    o_ref, S_ref = oracle.gdr_fwd(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("beta"),
                                  np64(x["S0"][:, h:h + 1]))
    assert max_rel(np64(o[:, :, h:h + 1]), o_ref) <= TOL_O["bf16"]
    assert fro_rel(np64(S_T[:, h:h + 1]), S_ref) <= TOL_S


def test_gdr_fwd_does_not_split_the_layer_workload():
    assert gdr.lib().gdr_fwd_workspace_bytes(4, 4096, 16, 128, 128, gdr.GDR_BF16) == 0
    assert gdr.lib().gdr_fwd_workspace_bytes(1, 1000, 16, 128, 128, gdr.GDR_BF16) == 0


@pytest.mark.parametrize("B,want_state", [(1, True), (1, False), (2, True)])
def test_split_forward_without_initial_state(B, want_state, monkeypatch):
    # S0 = 0: the first segment needs no correction, and with one batch no
    # identity pass either; outputs and the final state must still agree
    T, H = 8192, 8 if B == 1 else 4
    x = synth.gdr_inputs(B, T, H, 128, 128, "bf16", seed=20 + B)
    d = {n: dev(t) for n, t in x.items() if t is not None}
    assert gdr.lib().gdr_fwd_workspace_bytes(B, T, H, 128, 128, gdr.GDR_BF16) > 0
    o, S_T = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, return_state=want_state)
    monkeypatch.setenv("GDR_FWD_SPLIT", "off")
    o1, S1 = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None)
    gdr.check_status()
    assert max_rel(np64(o), np64(o1)) <= TOL_O["bf16"]
    if want_state:
        assert fro_rel(np64(S_T), np64(S1)) <= TOL_S
    else:
        assert S_T is None
    sl = lambda n: np64(x[n][:, :, 1:2])
    o_ref, _ = oracle.gdr_fwd(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("beta"), None)
    assert max_rel(np64(o[:, :, 1:2]), o_ref) <= TOL_O["bf16"]


def test_long_workload_forward_sampled_heads():
    # B1 T65536 H16 d128 bf16, S0 = 0: gdr_fwd runs it as two parallel
    # segments; the oracle follows two heads over all 65,536 tokens
    x = synth.workload_inputs("long_fwd_bwd")
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta")}
    o, S_T = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None)
    gdr.check_status()
    for h in (0, 9):
        sl = lambda n: np64(x[n][:, :, h:h + 1])
        o_ref, S_ref = oracle.gdr_fwd(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("beta"), None)
        assert max_rel(np64(o[:, :, h:h + 1]), o_ref) <= TOL_O["bf16"]
        assert fro_rel(np64(S_T[:, h:h + 1]), S_ref) <= TOL_S
