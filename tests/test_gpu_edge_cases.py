"""The method's degenerate and extreme cases on every GPU kernel that runs
the scalar-gate rule, against the fp64 oracle through the C ABI.

The cases follow the special cases the Gated DeltaNet review
(meaningful96.github.io/nr/GDN) singles out:

* ``alpha_one``: log alpha = 0, so alpha = 1 and the rule is DeltaNet
  (section 3.3; the gate of section 3.4 switched off).
* ``beta_zero``: beta = 0, no write: pure decay S_t = (prod alpha) S0
  (section 3.2, global forgetting).
* ``beta_one_unit_keys``: beta = 1 and q = k, unit keys: the delta rule's
  write-then-read, so o_t = S_t k_t returns v_t up to the rounding of the
  keys to the storage dtype (section 3.4).
* ``strong_decay``: log alpha = -1.5 on every token, so one 64-token chunk
  decays by e^-96, beyond the e^80 span where the cluster forward leaves
  its midpoint-referenced decay factors for exact exponentials.
* ``decay_spikes``: the usual gates with a few tokens at log alpha = -50,
  so some chunks take the exact branch and others do not.

Every case runs at bf16 d=128 over three full chunks and a ragged tail
(T = 229), on the two-SM cluster forward (default), the single-CTA tcgen05
forward (GDR_FWD_KERNEL=tc1), the CUDA-core forward (GDR_FWD_KERNEL=simt),
the sequence-split forward (a long sequence over few heads), the tcgen05
backward (default) and the CUDA-core backward (GDR_BWD_KERNEL=simt), and the
decode step.  Tolerances are those of the parity contract.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_91_b200 as gdr
import oracle
import synth
from gpu_common import TOL_G, TOL_O, TOL_S, dev, fro_rel, max_rel, np64

pytestmark = pytest.mark.gpu

CASES = ["alpha_one", "beta_zero", "beta_one_unit_keys", "strong_decay", "decay_spikes"]
B, T, H, D = 2, 229, 2, 128


def _case(name, T_=T, B_=B, H_=H, seed=0):
    """Seeded inputs of one edge case (bf16 q, k, v; fp32 gates; S0 ~ N(0, 0.02))."""
    x = synth.gdr_inputs(B_, T_, H_, D, D, "bf16", seed=1000 + seed + CASES.index(name),
                         s0_std=0.02, with_dO=True)
    if name == "alpha_one":
        x["log_alpha"] = torch.zeros_like(x["log_alpha"])
    elif name == "beta_zero":
        x["beta"] = torch.zeros_like(x["beta"])
    elif name == "beta_one_unit_keys":
        x["beta"] = torch.ones_like(x["beta"])
        x["q"] = x["k"].clone()
    elif name == "strong_decay":
        x["log_alpha"] = torch.full_like(x["log_alpha"], -1.5)
    elif name == "decay_spikes":
        la = x["log_alpha"].clone()
        la[:, 10] = -50.0          # chunk 0: span > 80 with the next spike
        la[:, 40] = -50.0
        la[:, (2 * T_) // 3] = -50.0  # a later chunk: one spike, span < 80 apart from it
        x["log_alpha"] = la
    return x


def _fwd_ref(x):
    a = {n: np64(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    return oracle.gdr_fwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["S0"])


def _fwd_gpu(x):
    return gdr.gdr_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]),
                       dev(x["beta"]), dev(x["S0"]))


def _check_fwd(x, o, ST):
    o_ref, ST_ref = _fwd_ref(x)
    o_np = np64(o)
    assert np.isfinite(o_np).all() and np.isfinite(np64(ST)).all()
    assert max_rel(o_np, o_ref) <= TOL_O["bf16"], max_rel(o_np, o_ref)
    assert fro_rel(np64(ST), ST_ref) <= TOL_S, fro_rel(np64(ST), ST_ref)
    return o_ref, ST_ref


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("kernel", ["default", "tc1", "simt"])
def test_fwd_edge_case(case, kernel, monkeypatch):
    if kernel != "default":
        monkeypatch.setenv("GDR_FWD_KERNEL", kernel)
    x = _case(case)
    o, ST = _fwd_gpu(x)
    gdr.check_status()
    o_ref, ST_ref = _check_fwd(x, o, ST)
    if case == "beta_one_unit_keys":
        # write-then-read: o_t = S_t k_t = v_t for exactly unit keys; the bf16
        # keys have |k|^2 = 1 + eps, |eps| < 2^-7, so o_t = v_t + O(eps)
        assert max_rel(np64(o), np64(x["v"])) <= TOL_O["bf16"]
    if case == "beta_zero":
        # pure decay: S_T = exp(sum log alpha) S0 per (b, h)
        decay = np.exp(np64(x["log_alpha"]).sum(axis=1))          # [B, H]
        closed = decay[:, :, None, None] * np64(x["S0"])
        assert fro_rel(np64(ST), closed) <= 1e-5


@pytest.mark.parametrize("case", CASES)
def test_split_forward_edge_case(case):
    """B1 H2 T4160 runs as two concurrent sequence segments joined by the
    scan of their affine maps and the tcgen05 correction."""
    x = _case(case, T_=4160, B_=1, H_=2, seed=7)
    ws = gdr.lib().gdr_fwd_workspace_bytes(1, 4160, 2, D, D, 1)  # 1 = bf16
    assert ws > 0, "this shape is expected to run as segments"
    o, ST = _fwd_gpu(x)
    gdr.check_status()
    _check_fwd(x, o, ST)


# Unit roundoff of a bf16 MMA operand: the tensor-core backward rounds every
# operand of its products (states, gradients of the state, keys, T'') to bf16.
U_BF16 = 2.0 ** -9


def _state_norms(a):
    """max over tokens and heads of |S_t|_F, by stepping the oracle (test only)."""
    S = np.ascontiguousarray(a["S0"].copy())
    worst = 0.0
    for t in range(a["q"].shape[1]):
        oracle.gdr_step_inplace(a["q"][:, t], a["k"][:, t], a["v"][:, t], a["log_alpha"][:, t],
                                a["beta"][:, t], S)
        worst = max(worst, float(np.sqrt((S ** 2).sum(axis=(2, 3))).max()))
    return worst


def _bwd_check(x, got, cancelling=False):
    a = {n: np64(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
    dST = np64(x["dST"])
    ref = oracle.gdr_bwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["S0"], a["dO"], dST)
    strict = ("dq", "dk", "dv", "dlog_alpha", "dbeta")
    if cancelling:
        strict = ("dq", "dk", "dv", "dbeta")
    for n in strict:
        g = np64(got[n])
        assert np.isfinite(g).all(), n
        assert max_rel(g, ref[n]) <= TOL_G["bf16"], (n, max_rel(g, ref[n]))
    if not cancelling:
        assert fro_rel(np64(got["dS0"]), ref["dS0"]) <= 1e-2
        return
    # beta = 1 with unit keys: every token erases its key direction, so the
    # gradient of the state shrinks from |dS_T| (12.8 here) to |dS0| (0.02)
    # and dlog alpha_t = alpha_t (<G_t, S_{t-1}> - r_t . de_t) is a small
    # difference of terms of size |G_t| |S_{t-1}|.  With bf16 operands the
    # error is bounded by the terms, not by the result: one product carries
    # at most 2u |G| |S| (both operands rounded), and dS0 picks up 4u |dS_T|
    # per chunk it crosses (dU = D K~^T, then D -= dU^T W: two products with
    # two rounded operands each).  The bounds are worst cases, well above the
    # typical error; the other cases hold the same outputs of the same kernel
    # to the parity tolerance.
    G = float(np.sqrt((dST ** 2).sum(axis=(2, 3))).max())
    nch = -(-a["q"].shape[1] // 64)
    gl = np64(got["dlog_alpha"])
    assert np.isfinite(gl).all()
    assert np.abs(gl - ref["dlog_alpha"]).max() <= 2 * U_BF16 * G * _state_norms(a)
    d0 = np64(got["dS0"]) - ref["dS0"]
    assert np.sqrt((d0 ** 2).sum(axis=(2, 3))).max() <= 4 * U_BF16 * nch * G


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("kernel", ["default", "simt"])
def test_bwd_edge_case(case, kernel, monkeypatch):
    """Both backward kernels against the oracle's reverse mode.  The fp32
    CUDA-core backward meets the parity tolerance in every case.  So does the
    bf16 tensor-core backward, except dlog alpha and dS0 in the write-then-
    read case: those results cancel, and they are held to the bound that the
    bf16 rounding of the MMA operands sets (see _bwd_check)."""
    if kernel != "default":
        monkeypatch.setenv("GDR_BWD_KERNEL", kernel)
    x = _case(case)
    x["dST"] = torch.randn(B, H, D, D, generator=torch.Generator().manual_seed(5)) * 0.05
    d = {n: dev(x[n]) for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO", "dST")}
    got = gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"], d["dST"])
    gdr.check_status()
    _bwd_check(x, got, cancelling=(case == "beta_one_unit_keys" and kernel == "default"))


@pytest.mark.parametrize("case", CASES)
def test_step_edge_case(case):
    """T decode steps from S0 equal the oracle's sequential forward at every
    token and in the final state."""
    x = _case(case, T_=100)
    o_ref, ST_ref = _fwd_ref(x)
    S = dev(x["S0"]).clone()
    worst = 0.0
    for t in range(100):
        ot = gdr.gdr_step(dev(x["q"][:, t]), dev(x["k"][:, t]), dev(x["v"][:, t]),
                          dev(x["log_alpha"][:, t]), dev(x["beta"][:, t]), S)
        worst = max(worst, max_rel(np64(ot), o_ref[:, t]))
    assert worst <= TOL_O["bf16"], worst
    assert fro_rel(np64(S), ST_ref) <= TOL_S
