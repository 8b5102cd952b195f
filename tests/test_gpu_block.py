"""GPU parity of the block prologue (ShortConv -> SiLU -> L2 on q, k; ShortConv
-> SiLU on v) and epilogue (RMSNorm * weight * SiLU(g)) against the fp64
oracle, through the C ABI.

Tolerance (elementwise; the pages state none for these steps): the kernels
compute in fp32 from the stored inputs and round once to the output dtype, so
|gpu - ref| <= 2^-8 |ref| + 2^-12 max|ref| for bf16 outputs (half an ulp of
bf16 is 2^-9 relative) and 1e-5 |ref| + 1e-6 max|ref| for fp32 outputs.  The
carried conv state is a copy of inputs and must match bit for bit."""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import dev, np64

pytestmark = pytest.mark.gpu


def assert_close(got, ref, dtype):
    got = np64(got) if isinstance(got, torch.Tensor) else np.asarray(got)
    ref = np.asarray(ref, dtype=np.float64)
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    if dtype == "bf16":
        bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * scale
    else:
        bound = 1e-5 * np.abs(ref) + 1e-6 * scale
    err = np.abs(got - ref)
    bad = err > bound
    assert not bad.any(), "%d of %d elements off; worst %.3e at %s (ref %.3e)" % (
        bad.sum(), bad.size, err.max(), np.unravel_index(np.argmax(err - bound), err.shape),
        ref.flat[np.argmax(err - bound)])


def oracle_prologue(x, eps):
    """Per-stream oracle results and the concatenated next conv state."""
    H, dk = x["xq"].shape[2], x["xq"].shape[3]
    st = x["conv_state"]
    outs, states = [], []
    off = 0
    for s, (xn, wn, bn) in enumerate((("xq", "wq", "bq"), ("xk", "wk", "bk"), ("xv", "wv", "bv"))):
        d = x[xn].shape[-1]
        sl = None if st is None else np64(st[:, :, off:off + H * d])
        y, so = oracle.short_conv(np64(x[xn]), np64(x[wn]), np64(x[bn]), sl, l2=s < 2, eps=eps)
        outs.append(y)
        states.append(so)
        off += H * d
    return outs, np.concatenate(states, axis=-1)


def run_prologue(x, eps, state_out=None, inplace=False):
    d = {k: dev(v) for k, v in x.items()}
    st = d["conv_state"]
    if inplace:
        state_out = st
    q, k, v = gdr.gdr_block_prologue(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["bq"],
                                     d["bk"], d["bv"], conv_state=st, conv_state_out=state_out,
                                     eps=eps)
    gdr.check_status()
    return q, k, v


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 3, 64, 130])
def test_prologue_small(dtype, dk, dv, T):
    B, H, K = 2, 3, 4
    x = synth.block_prologue_inputs(B, T, H, dk, dv, K, dtype, seed=T + dk + 7 * dv)
    ref, ref_state = oracle_prologue(x, 1e-6)
    so = torch.empty(B, K - 1, H * (2 * dk + dv), dtype=x["xq"].dtype, device="cuda")
    outs = run_prologue(x, 1e-6, state_out=so)
    for got, r in zip(outs, ref):
        assert_close(got, r, dtype)
    np.testing.assert_array_equal(np64(so), ref_state)


@pytest.mark.parametrize("K", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("bias,state", [(True, True), (False, False), (True, False)])
def test_prologue_conv_widths(K, bias, state):
    B, T, H, dk, dv = 2, 70, 2, 128, 128
    x = synth.block_prologue_inputs(B, T, H, dk, dv, K, "bf16", seed=K, bias=bias, state=state)
    ref, ref_state = oracle_prologue(x, 0.0)
    so = (torch.empty(B, K - 1, H * (2 * dk + dv), dtype=torch.bfloat16, device="cuda")
          if K > 1 else None)
    outs = run_prologue(x, 0.0, state_out=so)
    for got, r in zip(outs, ref):
        assert_close(got, r, "bf16")
    if K > 1:
        np.testing.assert_array_equal(np64(so), ref_state)


@pytest.mark.parametrize("T", [1, 2, 200])
def test_prologue_in_place_state(T):
    # conv_state_out == conv_state: decode (T = 1), T < K-1, and a long segment
    B, H, dk, dv, K = 3, 2, 128, 64, 4
    x = synth.block_prologue_inputs(B, T, H, dk, dv, K, "bf16", seed=100 + T)
    ref, ref_state = oracle_prologue(x, 1e-6)
    d = {k: dev(v) for k, v in x.items()}
    st = d["conv_state"]
    q, k, v = gdr.gdr_block_prologue(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["bq"],
                                     d["bk"], d["bv"], conv_state=st, conv_state_out=st, eps=1e-6)
    gdr.check_status()
    for got, r in zip((q, k, v), ref):
        assert_close(got, r, "bf16")
    np.testing.assert_array_equal(np64(st), ref_state)


def test_prologue_decode_chain_matches_one_pass():
    # A prefill of 37 tokens then 5 decode tokens through the carried state is
    # bit-identical to one pass over 42 tokens.
    B, H, dk, dv, K, T = 2, 4, 128, 128, 4, 42
    x = synth.block_prologue_inputs(B, T, H, dk, dv, K, "bf16", seed=5)
    d = {k: dev(v) for k, v in x.items()}
    full = gdr.gdr_block_prologue(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["bq"],
                                  d["bk"], d["bv"], conv_state=d["conv_state"], eps=1e-6)
    st = d["conv_state"].clone()
    pieces = [[], [], []]
    for a, b in [(0, 37)] + [(t, t + 1) for t in range(37, 42)]:
        xs = [d[n][:, a:b].contiguous() for n in ("xq", "xk", "xv")]
        outs = gdr.gdr_block_prologue(*xs, d["wq"], d["wk"], d["wv"], d["bq"], d["bk"], d["bv"],
                                      conv_state=st, conv_state_out=st, eps=1e-6)
        for i in range(3):
            pieces[i].append(outs[i])
    gdr.check_status()
    for i in range(3):
        assert torch.equal(torch.cat(pieces[i], dim=1), full[i])


def test_prologue_zero_input_gives_zero():
    B, T, H, d, K = 1, 5, 2, 128, 4
    z = torch.zeros(B, T, H, d, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(H * d, K, device="cuda")
    q, k, v = gdr.gdr_block_prologue(z, z, z, w, w, w, eps=1e-6)
    gdr.check_status()
    for t in (q, k, v):
        assert torch.count_nonzero(t) == 0


def test_prologue_workload_sampled_windows():
    # The full block shape (B4 T4096 H16 d128 bf16, K = 4) in the launch the
    # bench times; the oracle checks windows of tokens, each fed the K-1
    # preceding inputs as its carried state.
    B, T, H, dk, dv, K = 4, 4096, 16, 128, 128, 4
    x = synth.block_prologue_inputs(B, T, H, dk, dv, K, "bf16", seed=11, state=False)
    outs = run_prologue(x, 1e-6)
    for t0, L in ((0, 70), (1000, 40), (4096 - 67, 67)):
        for s, (xn, wn, bn) in enumerate((("xq", "wq", "bq"), ("xk", "wk", "bk"),
                                           ("xv", "wv", "bv"))):
            xs = np64(x[xn])
            st = None
            if t0 > 0:
                st = xs[:, t0 - (K - 1):t0].reshape(B, K - 1, -1)
            y, _ = oracle.short_conv(xs[:, t0:t0 + L], np64(x[wn]), np64(x[bn]), st, l2=s < 2,
                                     eps=1e-6)
            assert_close(outs[s][:, t0:t0 + L], y, "bf16")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("T", [1, 77])
def test_epilogue_small(dtype, dv, gate, T):
    x = synth.block_epilogue_inputs(2, T, 3, dv, dtype, seed=dv + T, gate=gate)
    ref = oracle.rmsnorm_gate(np64(x["o"]), np64(x["g"]), np64(x["weight"]), 1e-6)
    y = gdr.gdr_block_epilogue(dev(x["o"]), dev(x["g"]), dev(x["weight"]), 1e-6)
    gdr.check_status()
    assert_close(y, ref, dtype)


def test_epilogue_workload_full():
    x = synth.block_epilogue_inputs(4, 4096, 16, 128, "bf16", seed=3)
    ref = oracle.rmsnorm_gate(np64(x["o"]), np64(x["g"]), np64(x["weight"]), 1e-6)
    y = gdr.gdr_block_epilogue(dev(x["o"]), dev(x["g"]), dev(x["weight"]), 1e-6)
    gdr.check_status()
    assert_close(y, ref, "bf16")


def test_epilogue_zero_rows():
    o = torch.zeros(1, 3, 2, 128, dtype=torch.bfloat16, device="cuda")
    y = gdr.gdr_block_epilogue(o, torch.ones_like(o), torch.ones(128, device="cuda"), 1e-6)
    gdr.check_status()
    assert torch.count_nonzero(y) == 0


def _epi_bwd_ref(x, eps):
    return oracle.rmsnorm_gate_bwd(np64(x["o"]), np64(x["g"]), np64(x["weight"]), np64(x["dy"]), eps)


def _epi_bwd_gpu(x, eps):
    return gdr.gdr_block_epilogue_bwd(dev(x["o"]), dev(x["g"]), dev(x["weight"]), dev(x["dy"]), eps)


def _assert_dweight(got, ref, rows):
    # fp32 sums over `rows` rows: a relative bound that grows with the count
    scale = float(np.max(np.abs(ref)))
    err = float(np.max(np.abs(np64(got) - ref)))
    assert err <= (1e-5 + 2e-10 * rows) * scale, (err, scale)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("T", [1, 77, 300])
def test_epilogue_bwd_small(dtype, dv, gate, T):
    x = synth.block_epilogue_bwd_inputs(2, T, 3, dv, dtype, seed=dv + T + 5, gate=gate)
    ref = _epi_bwd_ref(x, 1e-6)
    do, dg, dw = _epi_bwd_gpu(x, 1e-6)
    gdr.check_status()
    assert_close(do, ref["do"], dtype)
    if gate:
        assert_close(dg, ref["dg"], dtype)
    else:
        assert dg is None
    _assert_dweight(dw, ref["dweight"], 2 * T * 3)


def test_epilogue_bwd_workload_full():
    # 262,144 rows: many 64-row units per block, every block's partial used
    x = synth.block_epilogue_bwd_inputs(4, 4096, 16, 128, "bf16", seed=4)
    ref = _epi_bwd_ref(x, 1e-6)
    do, dg, dw = _epi_bwd_gpu(x, 1e-6)
    gdr.check_status()
    assert_close(do, ref["do"], "bf16")
    assert_close(dg, ref["dg"], "bf16")
    _assert_dweight(dw, ref["dweight"], 4 * 4096 * 16)


def test_epilogue_bwd_is_deterministic():
    x = synth.block_epilogue_bwd_inputs(2, 3000, 8, 128, "bf16", seed=9)
    a = _epi_bwd_gpu(x, 1e-6)
    b = _epi_bwd_gpu(x, 1e-6)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_epilogue_bwd_zero_rows_and_large_eps():
    # o = 0: a = 0, so dg = 0 and do = dy weight SiLU(g) / sqrt(eps)
    x = synth.block_epilogue_bwd_inputs(1, 5, 2, 128, "f32", seed=2)
    x["o"] = torch.zeros_like(x["o"])
    ref = _epi_bwd_ref(x, 0.25)
    do, dg, dw = _epi_bwd_gpu(x, 0.25)
    gdr.check_status()
    assert torch.count_nonzero(dg) == 0 and torch.count_nonzero(dw) == 0
    assert_close(do, ref["do"], "f32")


def _stream_cols(H, dk, dv):
    return ((0, H * dk), (H * dk, 2 * H * dk), (2 * H * dk, H * (2 * dk + dv)))


def _pro_bwd_ref(x, eps):
    """Oracle reverse mode per stream; states split by column."""
    H, dk, dv = x["xq"].shape[2], x["xq"].shape[3], x["xv"].shape[3]
    st, dso = x["conv_state"], x["dconv_state_out"]
    refs = []
    for i, (s, (a_, b_)) in enumerate(zip("qkv", _stream_cols(H, dk, dv))):
        refs.append(oracle.short_conv_bwd(
            np64(x["x" + s]), np64(x["w" + s]), np64(x["dy" + s]), np64(x["b" + s]),
            None if st is None else np64(st)[:, :, a_:b_], None if dso is None else np64(dso)[:, :, a_:b_],
            l2=i < 2, eps=eps))
    return refs


def _pro_bwd_gpu(x, eps, want_dconv_state=None):
    d = {k: dev(v) for k, v in x.items()}
    out = gdr.gdr_block_prologue_bwd(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["dyq"], d["dyk"],
                                     d["dyv"], d["bq"], d["bk"], d["bv"], conv_state=d["conv_state"],
                                     dconv_state_out=d["dconv_state_out"], eps=eps,
                                     want_dconv_state=want_dconv_state)
    gdr.check_status()
    return out


def _check_pro_bwd(x, out, refs, dtype):
    B, T, H, dk = x["xq"].shape
    dv = x["xv"].shape[3]
    for s, r, (a_, b_) in zip("qkv", refs, _stream_cols(H, dk, dv)):
        assert_close(out["dx" + s], r["dx"], dtype)
        _assert_dweight(out["dw" + s], r["dw"], B * T)
        if out["db" + s] is not None:
            _assert_dweight(out["db" + s], r["dbias"], B * T)
        if out["dconv_state"] is not None:
            assert_close(out["dconv_state"][:, :, a_:b_], r["dstate"], dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 3, 64, 130])
def test_prologue_bwd_small(dtype, dk, dv, T):
    x = synth.block_prologue_bwd_inputs(2, T, 3, dk, dv, 4, dtype, seed=T + dk + 5 * dv, dstate=True)
    _check_pro_bwd(x, _pro_bwd_gpu(x, 1e-6), _pro_bwd_ref(x, 1e-6), dtype)


@pytest.mark.parametrize("K", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("bias,state,dstate", [(True, True, True), (False, False, False), (True, False, True),
                                              (False, True, False)])
def test_prologue_bwd_widths_and_optional_inputs(K, bias, state, dstate):
    x = synth.block_prologue_bwd_inputs(2, 97, 2, 128, 128, K, "bf16", seed=K * 11 + bias + 2 * state,
                                        bias=bias, state=state, dstate=dstate)
    _check_pro_bwd(x, _pro_bwd_gpu(x, 1e-6, want_dconv_state=K > 1), _pro_bwd_ref(x, 1e-6), "bf16")


@pytest.mark.parametrize("K", [4, 8])
@pytest.mark.parametrize("T", [1, 2, 5])
@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128)])
def test_prologue_bwd_shorter_than_the_window(T, K, dtype, d):
    # T < K-1 (and, at K = 4, T >= K-1 for T = 5): part of the returned state
    # is the carried-in state, so the gradient of the returned state flows
    # into dconv_state_in; both the carried state and that gradient are given
    x = synth.block_prologue_bwd_inputs(1, T, 2, d, d, K, dtype, seed=T + 10 * K, state=True, dstate=True)
    assert x["conv_state"] is not None and x["dconv_state_out"] is not None
    eps = 0.0 if dtype == "f32" else 1e-6
    _check_pro_bwd(x, _pro_bwd_gpu(x, eps), _pro_bwd_ref(x, eps), dtype)


@pytest.mark.parametrize("K", [3, 4, 8])
def test_prologue_bwd_blocks_walk_several_runs(K):
    # H16 gives 48 (stream, head) pairs and a few blocks per pair, so a block
    # walks several 64-token runs from the last to the first, carrying the
    # dz rows of each run's first tokens to the run before it.  At B4 T700
    # (11 runs, the last of 60 tokens) some blocks' ranges cross a batch
    # boundary, where the carried rows must be zero.
    x = synth.block_prologue_bwd_inputs(4, 700, 16, 128, 128, K, "bf16", seed=40 + K, state=True, dstate=True)
    _check_pro_bwd(x, _pro_bwd_gpu(x, 1e-6, want_dconv_state=True), _pro_bwd_ref(x, 1e-6), "bf16")


def test_prologue_bwd_workload_full():
    # B4 T4096 H16 d128 K4 bf16: every element of dx and the full sums
    x = synth.block_prologue_bwd_inputs(4, 4096, 16, 128, 128, 4, "bf16", seed=31, state=False)
    out = _pro_bwd_gpu(x, 1e-6)
    refs = _pro_bwd_ref(x, 1e-6)
    _check_pro_bwd(x, out, refs, "bf16")


def test_prologue_bwd_is_deterministic():
    x = synth.block_prologue_bwd_inputs(2, 1500, 8, 128, 128, 4, "bf16", seed=3, dstate=True)
    a = _pro_bwd_gpu(x, 1e-6)
    b = _pro_bwd_gpu(x, 1e-6)
    for n in a:
        if a[n] is not None:
            assert torch.equal(a[n], b[n]), n


def test_block_kernels_count_launches():
    x = synth.block_prologue_inputs(1, 10, 1, 64, 64, 4, "bf16", seed=1)
    before = gdr.launch_count()
    run_prologue(x, 1e-6)
    e = synth.block_epilogue_inputs(1, 10, 1, 64, "bf16", seed=1)
    gdr.gdr_block_epilogue(dev(e["o"]), dev(e["g"]), dev(e["weight"]))
    assert gdr.launch_count() - before == 2
    e["dy"] = torch.ones_like(e["o"])
    _epi_bwd_gpu(e, 1e-6)   # the backward and its fixed-order dweight sum
    assert gdr.launch_count() - before == 4
    _pro_bwd_gpu(synth.block_prologue_bwd_inputs(1, 10, 1, 64, 64, 4, "bf16", seed=1), 1e-6)
    assert gdr.launch_count() - before == 6
