"""The autograd bindings (gradients through the library's backward calls,
checked against the fp64 oracle's reverse mode) and CUDA-graph capture of
library calls (a captured decode loop and forward replay to the same
results as eager calls)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gated_delta_rule_91_b200.autograd import block_epilogue, block_prologue, gated_delta_rule, gated_delta_rule2
from gpu_common import TOL_G, TOL_O, dtype_name, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu


def _leaf(t):
    return None if t is None else t.cuda().requires_grad_(True)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_autograd_matches_oracle_reverse_mode(dtype, d):
    x = synth.gdr_inputs(2, 150, 2, d, d, dtype, seed=3, s0_std=0.02)
    leaves = {n: _leaf(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    o, S_T = gated_delta_rule(*(leaves[n] for n in ("q", "k", "v", "log_alpha", "beta", "S0")))
    g = torch.Generator().manual_seed(1)
    wo = torch.randn(o.shape, generator=g).to(o.dtype).cuda()
    ws = torch.randn(S_T.shape, generator=g).cuda()
    ((o.float() * wo.float()).sum() + (S_T * ws).sum()).backward()
    ref = oracle.gdr_bwd(np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["log_alpha"]), np64(x["beta"]),
                         np64(x["S0"]), np64(wo), np64(ws))
    tol = TOL_G[dtype_name(leaves["q"])]
    for n, rn in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_alpha", "dlog_alpha"), ("beta", "dbeta")):
        assert max_rel(np64(leaves[n].grad), ref[rn]) <= tol, n
    assert fro_rel(np64(leaves["S0"].grad), ref["dS0"]) <= (1e-2 if dtype == "bf16" else 1e-4)


def test_autograd_gdn2_and_unused_state():
    x = synth.gdr2_inputs(1, 100, 2, 128, 128, "bf16", seed=5, s0_std=0.02)
    leaves = {n: _leaf(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}
    o, _ = gated_delta_rule2(*(leaves[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")))
    wo = torch.randn(o.shape, generator=torch.Generator().manual_seed(2)).to(o.dtype).cuda()
    (o.float() * wo.float()).sum().backward()   # S_T unused: a zero gradient reaches gdr2_bwd
    ref = oracle.gdr2_bwd(np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["log_alpha"]), np64(x["b"]),
                          np64(x["w"]), np64(x["S0"]), np64(wo))
    for n, rn in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_alpha", "dlog_alpha"), ("b", "db"),
                  ("w", "dw")):
        assert max_rel(np64(leaves[n].grad), ref[rn]) <= TOL_G["bf16"], n


def test_autograd_without_initial_state():
    x = synth.gdr_inputs(1, 70, 2, 64, 64, "f32", seed=6)
    leaves = {n: _leaf(x[n]) for n in ("q", "k", "v", "log_alpha", "beta")}
    o, S_T = gated_delta_rule(*(leaves[n] for n in ("q", "k", "v", "log_alpha", "beta")), None)
    (o.sum() + S_T.sum()).backward()
    ref = oracle.gdr_bwd(np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["log_alpha"]), np64(x["beta"]),
                         None, np.ones(o.shape), np.ones(S_T.shape))
    assert max_rel(np64(leaves["k"].grad), ref["dk"]) <= TOL_G["f32"]


@pytest.mark.parametrize("gate", [True, False])
def test_autograd_block_epilogue(gate):
    x = synth.block_epilogue_bwd_inputs(2, 90, 3, 128, "bf16", seed=11, gate=gate)
    o, w = _leaf(x["o"]), _leaf(x["weight"])
    g = _leaf(x["g"])
    y = block_epilogue(o, g, w, 1e-6)
    (y.float() * x["dy"].cuda().float()).sum().backward()
    ref = oracle.rmsnorm_gate_bwd(np64(x["o"]), np64(x["g"]), np64(x["weight"]), np64(x["dy"]), 1e-6)
    assert max_rel(np64(o.grad), ref["do"]) <= TOL_O["bf16"]
    assert max_rel(np64(w.grad), ref["dweight"]) <= 1e-4
    if gate:
        assert max_rel(np64(g.grad), ref["dg"]) <= TOL_O["bf16"]


def test_autograd_block_prologue_into_the_rule():
    # prologue -> gated delta rule, one loss: gradients reach the conv taps,
    # biases, inputs and the carried conv state through both backward calls
    B, T, H, d, K = 1, 80, 2, 128, 4
    px = synth.block_prologue_inputs(B, T, H, d, d, K, "bf16", seed=12)
    gx = synth.gdr_inputs(B, T, H, d, d, "bf16", seed=13)
    leaves = {n: _leaf(t) for n, t in px.items()}
    q, k, v = block_prologue(*(leaves[n] for n in ("xq", "xk", "xv", "wq", "wk", "wv", "bq", "bk", "bv",
                                                   "conv_state")), eps=1e-6)
    la, be = gx["log_alpha"].cuda(), gx["beta"].cuda()
    o, _ = gated_delta_rule(q, k, v, la, be, None)
    wo = torch.randn(o.shape, generator=torch.Generator().manual_seed(3)).to(o.dtype).cuda()
    (o.float() * wo.float()).sum().backward()
    # reference: the oracle's forward of both steps, then both reverse modes
    cols = ((0, H * d), (H * d, 2 * H * d), (2 * H * d, 3 * H * d))
    ys = []
    for i, (s, (a_, b_)) in enumerate(zip("qkv", cols)):
        y, _ = oracle.short_conv(np64(px["x" + s]), np64(px["w" + s]), np64(px["b" + s]),
                                 np64(px["conv_state"])[:, :, a_:b_], l2=i < 2, eps=1e-6)
        ys.append(y)
    # the rule consumes bf16 q, k, v: round the oracle's prologue outputs the same way
    ys = [torch.from_numpy(y).to(torch.bfloat16).double().numpy() for y in ys]
    gr = oracle.gdr_bwd(ys[0], ys[1], ys[2], np64(gx["log_alpha"]), np64(gx["beta"]), None, np64(wo),
                        np.zeros((B, H, d, d)))
    for i, (s, (a_, b_)) in enumerate(zip("qkv", cols)):
        ref = oracle.short_conv_bwd(np64(px["x" + s]), np64(px["w" + s]), gr["d" + s], np64(px["b" + s]),
                                    np64(px["conv_state"])[:, :, a_:b_], l2=i < 2, eps=1e-6)
        assert max_rel(np64(leaves["x" + s].grad), ref["dx"]) <= TOL_G["bf16"], s
        assert max_rel(np64(leaves["w" + s].grad), ref["dw"]) <= TOL_G["bf16"], s
        assert max_rel(np64(leaves["b" + s].grad), ref["dbias"]) <= TOL_G["bf16"], s
        assert max_rel(np64(leaves["conv_state"].grad)[:, :, a_:b_], ref["dstate"]) <= TOL_G["bf16"], s


def test_captured_decode_loop_replays_like_eager():
    B, H, d, steps = 8, 4, 128, 10
    S0 = synth.decode_state(B, H, d, d, seed=1).cuda()
    xs = [{n: t.cuda() for n, t in synth.decode_step_inputs(B, H, d, d, "bf16", 1, s).items()} for s in range(steps)]
    # eager
    S_e = S0.clone()
    o_e = [gdr.gdr_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_e) for x in xs]
    # captured on a side stream, then replayed from the same starting state
    S_g = S0.clone()
    outs = [torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(steps)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):   # warm-up outside the capture (kernel attributes)
        gdr.gdr_step(xs[0]["q"], xs[0]["k"], xs[0]["v"], xs[0]["log_alpha"], xs[0]["beta"], S_g.clone())
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for x, out in zip(xs, outs):
            gdr.gdr_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_g, o=out)
    S_g.copy_(S0)
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs, o_e):
        assert torch.equal(a, b)
    assert torch.equal(S_g, S_e)


def test_captured_forward_replays_like_eager():
    x = synth.gdr_inputs(2, 300, 4, 128, 128, "bf16", seed=8, s0_std=0.02)
    d = {n: t.cuda() for n, t in x.items() if t is not None}
    o_e, S_e = gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    o = torch.empty_like(o_e)
    S_T = torch.empty_like(S_e)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], o=o, S_T=S_T)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_e)
    assert torch.equal(S_T, S_e)
    assert max_rel(np64(o), np64(o_e)) <= TOL_O["bf16"]
