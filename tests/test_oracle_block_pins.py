"""Pins for the block oracle (oracle.short_conv, oracle.rmsnorm_gate): the
Gated DeltaNet block's ShortConv -> SiLU -> L2 prologue and RMSNorm -> SiLU
output-gate epilogue, checked against numpy/torch library routines on the
special cases that reduce to them, impulse responses, continuity of the
carried conv state, invariants and closed forms (CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle


def _silu_lib(z):
    return torch.nn.functional.silu(torch.from_numpy(np.asarray(z, dtype=np.float64))).numpy()


@pytest.mark.parametrize("K", [1, 2, 4, 7])
def test_zero_state_conv_is_numpy_convolution(K):
    # Zero carried state + no bias: each channel is a causal FIR filter, which
    # np.convolve computes with the filter taps reversed (cross-correlation).
    rng = np.random.default_rng(10 + K)
    B, T, H, d = 2, 19, 3, 8
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((H * d, K))
    y, _ = oracle.short_conv(x, w)
    xf = x.reshape(B, T, H * d)
    z = np.empty_like(xf)
    for b in range(B):
        for c in range(H * d):
            z[b, :, c] = np.convolve(xf[b, :, c], w[c, ::-1])[:T]
    np.testing.assert_allclose(y.reshape(B, T, H * d), _silu_lib(z), rtol=1e-13, atol=1e-14)


def test_conv_matches_torch_conv1d_with_bias_and_state():
    # A carried state is the same as prepending it to the sequence: torch's
    # depthwise conv1d (groups = channels) over the concatenation, bias added.
    rng = np.random.default_rng(3)
    B, T, H, d, K = 2, 11, 2, 16, 4
    C = H * d
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((C, K))
    bias = rng.standard_normal(C)
    st = rng.standard_normal((B, K - 1, C))
    y, _ = oracle.short_conv(x, w, bias, st)
    seq = np.concatenate([st, x.reshape(B, T, C)], axis=1)  # [B, K-1+T, C]
    z = torch.nn.functional.conv1d(torch.from_numpy(seq).transpose(1, 2),
                                   torch.from_numpy(w).unsqueeze(1), torch.from_numpy(bias),
                                   groups=C)  # valid convolution: T outputs
    ref = torch.nn.functional.silu(z).transpose(1, 2).numpy()
    np.testing.assert_allclose(y.reshape(B, T, C), ref, rtol=1e-13, atol=1e-14)


def test_impulse_response_reads_taps_in_reverse():
    # x = delta at token t0 in one channel: the pre-activation at t0 + m is
    # w[c, K-1-m]; everything else is silu(0) = 0.
    B, T, H, d, K = 1, 12, 1, 4, 4
    w = np.arange(1, H * d * K + 1, dtype=np.float64).reshape(H * d, K) / 10.0
    x = np.zeros((B, T, H, d))
    t0, c = 5, 2
    x[0, t0, 0, c] = 1.0
    y, _ = oracle.short_conv(x, w)
    expect = np.zeros((T, d))
    for m in range(K):
        expect[t0 + m, c] = w[c, K - 1 - m] / (1.0 + math.exp(-w[c, K - 1 - m]))
    np.testing.assert_allclose(y[0, :, 0, :], expect, rtol=1e-15, atol=0)


def test_impulse_in_carried_state():
    # An impulse in the carried state's oldest slot (token -(K-1)) only reaches
    # output token 0, through tap 0.
    B, T, H, d, K = 1, 6, 1, 2, 4
    w = np.array([[0.5, -1.0, 2.0, 3.0], [1.5, 0.25, -2.0, 1.0]])
    st = np.zeros((B, K - 1, H * d))
    st[0, 0, 1] = 1.0
    y, _ = oracle.short_conv(np.zeros((B, T, H, d)), w, state=st)
    expect = np.zeros((T, d))
    expect[0, 1] = 1.5 / (1.0 + math.exp(-1.5))
    np.testing.assert_allclose(y[0, :, 0, :], expect, rtol=1e-15, atol=0)


@pytest.mark.parametrize("t1", [0, 1, 2, 3, 9, 20])
@pytest.mark.parametrize("l2", [False, True])
def test_carried_state_makes_segments_continuous(t1, l2):
    # Running [0, t1) then [t1, T) with the carried state equals one run,
    # including segments shorter than K-1 tokens.
    rng = np.random.default_rng(t1)
    B, T, H, d, K = 2, 20, 2, 8, 4
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((H * d, K))
    bias = rng.standard_normal(H * d)
    s0 = rng.standard_normal((B, K - 1, H * d))
    y, sT = oracle.short_conv(x, w, bias, s0, l2=l2, eps=1e-6)
    ya, sa = oracle.short_conv(x[:, :t1], w, bias, s0, l2=l2, eps=1e-6) if t1 else (x[:, :0], s0)
    yb, sb = oracle.short_conv(x[:, t1:], w, bias, sa, l2=l2, eps=1e-6)
    np.testing.assert_array_equal(np.concatenate([ya, yb], axis=1), y)
    np.testing.assert_array_equal(sb, sT)


def test_state_out_is_last_inputs():
    rng = np.random.default_rng(5)
    B, T, H, d, K = 2, 2, 1, 4, 4  # T < K-1: the old state shifts in
    x = rng.standard_normal((B, T, H, d))
    s0 = rng.standard_normal((B, K - 1, H * d))
    _, s1 = oracle.short_conv(x, np.ones((d, K)), state=s0)
    np.testing.assert_array_equal(s1[:, 0], s0[:, 2])
    np.testing.assert_array_equal(s1[:, 1:], x.reshape(B, T, d))


def test_silu_closed_forms_through_identity_filter():
    # Filter = last tap only: y = silu(x).  silu(0) = 0, silu(ln 3) = (3/4) ln 3,
    # silu(-z) = silu(z) - z, silu(z) -> z for large z.
    K, d = 4, 4
    w = np.zeros((d, K))
    w[:, K - 1] = 1.0
    z = np.array([0.0, math.log(3.0), 2.5, 40.0])
    y, _ = oracle.short_conv(z.reshape(1, 1, 1, d), w)
    assert y[0, 0, 0, 0] == 0.0
    assert abs(y[0, 0, 0, 1] - 0.75 * math.log(3.0)) < 1e-15
    assert abs(y[0, 0, 0, 3] - 40.0) < 1e-15
    yn, _ = oracle.short_conv(-z.reshape(1, 1, 1, d), w)
    np.testing.assert_allclose(yn[0, 0, 0], y[0, 0, 0] - z, rtol=0, atol=1e-14)


def test_bias_alone():
    d, K = 8, 4
    bias = np.linspace(-3, 3, d)
    y, _ = oracle.short_conv(np.zeros((1, 3, 1, d)), np.ones((d, K)), bias)
    for t in range(3):
        np.testing.assert_allclose(y[0, t, 0], _silu_lib(bias), rtol=1e-15)


def test_l2_gives_unit_norm_per_head_and_keeps_direction():
    rng = np.random.default_rng(7)
    B, T, H, d, K = 2, 9, 3, 16, 4
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((H * d, K))
    y, _ = oracle.short_conv(x, w)
    yn, _ = oracle.short_conv(x, w, l2=True)
    np.testing.assert_allclose(np.linalg.norm(yn, axis=-1), 1.0, rtol=1e-14)
    # same direction: yn = y / |y| with a positive factor per (token, head)
    ratio = yn / y
    np.testing.assert_allclose(ratio, np.broadcast_to(ratio[..., :1], ratio.shape), rtol=1e-12)
    assert (ratio > 0).all()
    # with eps the norm is sqrt(s / (s + eps))
    eps = 0.3
    ye, _ = oracle.short_conv(x, w, l2=True, eps=eps)
    s = (y ** 2).sum(-1)
    np.testing.assert_allclose(np.linalg.norm(ye, axis=-1), np.sqrt(s / (s + eps)), rtol=1e-13)


def test_rmsnorm_constant_vector_and_mean_not_sum():
    # o = c * 1: mean(o^2) = c^2, so y = sign(c) * weight (eps = 0); a sum
    # instead of a mean would give weight / sqrt(dv).
    dv = 32
    o = np.zeros((1, 2, 2, dv))
    o[0, 0, 0] = 3.0
    o[0, 0, 1] = -0.5
    o[0, 1, 0] = 1e-3
    o[0, 1, 1] = 7.0
    wgt = np.linspace(0.5, 2.0, dv)
    y = oracle.rmsnorm_gate(o, None, wgt)
    sign = np.sign(o[..., :1])
    np.testing.assert_allclose(y, sign * wgt, rtol=1e-15)
    # eps: y = c / sqrt(c^2 + eps) * weight
    ye = oracle.rmsnorm_gate(o, None, wgt, eps=0.25)
    c = o[..., :1]
    np.testing.assert_allclose(ye, c / np.sqrt(c * c + 0.25) * wgt, rtol=1e-15)


def test_rmsnorm_invariants():
    rng = np.random.default_rng(11)
    o = rng.standard_normal((2, 5, 3, 64))
    ones = np.ones(64)
    y = oracle.rmsnorm_gate(o, None, ones)
    np.testing.assert_allclose((y ** 2).mean(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(oracle.rmsnorm_gate(4.5 * o, None, ones), y, rtol=1e-14)
    np.testing.assert_allclose(oracle.rmsnorm_gate(-o, None, ones), -y, rtol=1e-15)


def test_output_gate_closed_forms():
    rng = np.random.default_rng(12)
    o = rng.standard_normal((1, 4, 2, 16))
    wgt = rng.uniform(0.5, 1.5, 16)
    plain = oracle.rmsnorm_gate(o, None, wgt)
    assert (oracle.rmsnorm_gate(o, np.zeros_like(o), wgt) == 0).all()     # silu(0) = 0
    g3 = np.full_like(o, math.log(3.0))                                   # silu(ln 3)
    np.testing.assert_allclose(oracle.rmsnorm_gate(o, g3, wgt), plain * 0.75 * math.log(3.0),
                               rtol=1e-14)
    g = rng.standard_normal(o.shape)                                      # library SiLU
    np.testing.assert_allclose(oracle.rmsnorm_gate(o, g, wgt), plain * _silu_lib(g), rtol=1e-13)


def _fd(f, x, eps=1e-6):
    """Central finite differences of the scalar f at x (array), elementwise."""
    gr = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        xp = x.copy(); xp[idx] += eps
        xm = x.copy(); xm[idx] -= eps
        gr[idx] = (f(xp) - f(xm)) / (2 * eps)
    return gr


@pytest.mark.parametrize("gate,eps", [(True, 1e-6), (False, 0.0), (True, 0.3)])
def test_rmsnorm_gate_bwd_matches_finite_differences(gate, eps):
    rng = np.random.default_rng(30 + int(gate))
    o = rng.standard_normal((1, 2, 2, 6))
    g = rng.standard_normal(o.shape) if gate else None
    wgt = rng.uniform(0.5, 1.5, 6)
    dy = rng.standard_normal(o.shape)
    loss = lambda o_, g_, w_: float((oracle.rmsnorm_gate(o_, g_, w_, eps) * dy).sum())
    got = oracle.rmsnorm_gate_bwd(o, g, wgt, dy, eps)
    np.testing.assert_allclose(got["do"], _fd(lambda v: loss(v, g, wgt), o), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(got["dweight"], _fd(lambda v: loss(o, g, v), wgt), rtol=1e-6, atol=1e-8)
    if gate:
        np.testing.assert_allclose(got["dg"], _fd(lambda v: loss(o, v, wgt), g), rtol=1e-6, atol=1e-8)
    else:
        assert got["dg"] is None


def test_rmsnorm_bwd_is_orthogonal_to_the_row():
    # with eps = 0 the norm is scale-invariant, so do . o = 0 per row
    rng = np.random.default_rng(4)
    o = rng.standard_normal((2, 3, 2, 16))
    got = oracle.rmsnorm_gate_bwd(o, rng.standard_normal(o.shape), np.ones(16), rng.standard_normal(o.shape))
    np.testing.assert_allclose((got["do"] * o).sum(-1), 0.0, atol=1e-12)


def _conv_loss(x, w, bias, st, dy, dso, l2, eps):
    y, so = oracle.short_conv(x, w, bias, st, l2=l2, eps=eps)
    return float((y * dy).sum() + ((so * dso).sum() if dso is not None else 0.0))


@pytest.mark.parametrize("K,T,l2,eps", [(4, 6, True, 1e-6), (4, 2, True, 0.3), (3, 5, False, 0.0),
                                         (1, 4, True, 0.0), (2, 1, False, 0.0)])
def test_short_conv_bwd_matches_finite_differences(K, T, l2, eps):
    rng = np.random.default_rng(40 + K + T)
    B, H, d = 2, 2, 3
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((H * d, K))
    bias = rng.standard_normal(H * d)
    st = rng.standard_normal((B, K - 1, H * d))
    dy = rng.standard_normal(x.shape)
    dso = rng.standard_normal((B, K - 1, H * d))
    got = oracle.short_conv_bwd(x, w, dy, bias, st, dso, l2=l2, eps=eps)
    f = lambda **kw: _conv_loss(**{**dict(x=x, w=w, bias=bias, st=st, dy=dy, dso=dso, l2=l2, eps=eps), **kw})
    np.testing.assert_allclose(got["dx"], _fd(lambda v: f(x=v), x), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(got["dw"], _fd(lambda v: f(w=v), w), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(got["dbias"], _fd(lambda v: f(bias=v), bias), rtol=1e-6, atol=1e-8)
    if K > 1:
        np.testing.assert_allclose(got["dstate"], _fd(lambda v: f(st=v), st), rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("l2", [False, True])
def test_short_conv_bwd_matches_torch_autograd(l2):
    # torch's depthwise conv1d over [state, x], SiLU and F.normalize (eps
    # inside the norm's clamp is 0 here), differentiated by torch autograd.
    rng = np.random.default_rng(8)
    B, T, H, d, K = 2, 9, 2, 8, 4
    C = H * d
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((C, K))
    bias = rng.standard_normal(C)
    st = rng.standard_normal((B, K - 1, C))
    dy = rng.standard_normal(x.shape)
    tx, tw, tb, ts = (torch.tensor(a, requires_grad=True) for a in (x, w, bias, st))
    seq = torch.cat([ts, tx.reshape(B, T, C)], dim=1)
    z = torch.nn.functional.conv1d(seq.transpose(1, 2), tw.unsqueeze(1), tb, groups=C).transpose(1, 2)
    u = torch.nn.functional.silu(z).reshape(B, T, H, d)
    y = torch.nn.functional.normalize(u, dim=-1, eps=0.0) if l2 else u
    (y * torch.from_numpy(dy)).sum().backward()
    got = oracle.short_conv_bwd(x, w, dy, bias, st, l2=l2)
    np.testing.assert_allclose(got["dx"], tx.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(got["dw"], tw.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(got["dbias"], tb.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(got["dstate"], ts.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_short_conv_bwd_l2_is_orthogonal_to_the_row():
    # with eps = 0 the L2 output is scale-invariant in u: du . u = 0 per head
    # row, so with an identity filter (last tap 1, no bias) dz / silu'(x) . silu(x) = 0
    rng = np.random.default_rng(9)
    B, T, H, d, K = 1, 4, 2, 8, 3
    x = rng.standard_normal((B, T, H, d))
    w = np.zeros((H * d, K))
    w[:, K - 1] = 1.0
    got = oracle.short_conv_bwd(x, w, rng.standard_normal(x.shape), l2=True)
    sig = 1.0 / (1.0 + np.exp(-x))
    du = got["dx"] / (sig * (1.0 + x * (1.0 - sig)))
    np.testing.assert_allclose((du * x * sig).sum(-1), 0.0, atol=1e-12)
