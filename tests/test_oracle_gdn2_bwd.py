"""Pins of the oracle's Gated DeltaNet-2 backward (CPU only, fp64).

The pages give no backward; oracle.gdr2_bwd is the reverse mode of the
Gated Delta Rule-2 step ("Gated DeltaNet-2: Decoupling Erase and Write in
Linear Attention", agihunt.info/papers/2605.22791, the Gated Delta Rule-2
paragraph).  Checks:
  * central finite differences of L = <o, dO> + <S_T, dS_T> for every input
    (q, k, v, log alpha, b, w, S0), on a short sequence and, sampled, on one
    that crosses the oracle's 64-token checkpoint boundary;
  * collapse to the scalar-gate rule: b = w = beta*1 and a scalar decay give
    the gated delta rule's gradients, with dlog alpha summed over channels
    and dbeta = sum_j db_j + sum_i dw_i.
"""
import numpy as np
import pytest

import oracle
from pins_common import rand_inputs, rel_err


def _inputs(rng, B, T, H, dk, dv):
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk)) / np.sqrt(dk)
    v = rng.normal(size=(B, T, H, dv))
    la = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(B, T, H, dk))))
    b = rng.uniform(0.0, 2.0, size=(B, T, H, dk))
    w = rng.uniform(0.0, 1.0, size=(B, T, H, dv))
    S0 = rng.normal(size=(B, H, dv, dk)) * 0.5
    dO = rng.normal(size=(B, T, H, dv))
    dST = rng.normal(size=(B, H, dv, dk))
    return dict(q=q, k=k, v=v, la=la, b=b, w=w, S0=S0), dO, dST


NAMES = dict(q="dq", k="dk", v="dv", la="dlog_alpha", b="db", w="dw", S0="dS0")


def _loss(a, dO, dST):
    o, S = oracle.gdr2_fwd(a["q"], a["k"], a["v"], a["la"], a["b"], a["w"], a["S0"])
    return float((o * dO).sum() + (S * dST).sum())


def _check_fd(a, dO, dST, per_input=None, seed=0):
    g = oracle.gdr2_bwd(a["q"], a["k"], a["v"], a["la"], a["b"], a["w"], a["S0"], dO, dST)
    rng = np.random.default_rng(seed)
    eps = 1e-6
    for n, x in a.items():
        idx_all = list(np.ndindex(x.shape))
        if per_input is not None:
            pick = rng.choice(len(idx_all), size=min(per_input, len(idx_all)), replace=False)
            idx_all = [idx_all[i] for i in pick]
        for idx in idx_all:
            ap = {m: y.copy() for m, y in a.items()}
            ap[n][idx] += eps
            lp = _loss(ap, dO, dST)
            ap[n][idx] -= 2 * eps
            lm = _loss(ap, dO, dST)
            num = (lp - lm) / (2 * eps)
            got = g[NAMES[n]][idx]
            assert abs(num - got) <= 1e-6 * max(1.0, abs(num)), (n, idx, num, got)


def test_bwd_matches_finite_differences():
    a, dO, dST = _inputs(np.random.default_rng(60), 1, 6, 2, 4, 3)
    _check_fd(a, dO, dST)


def test_bwd_finite_differences_across_a_checkpoint_boundary():
    a, dO, dST = _inputs(np.random.default_rng(61), 1, 70, 1, 3, 2)
    _check_fd(a, dO, dST, per_input=12, seed=1)


def test_bwd_collapses_to_gated_delta_rule():
    rng = np.random.default_rng(62)
    B, T, H, dk, dv = 2, 40, 2, 5, 4
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    dO = rng.normal(size=(B, T, H, dv))
    dST = rng.normal(size=(B, H, dv, dk))
    g2 = oracle.gdr2_bwd(q, k, v, np.repeat(la[..., None], dk, axis=-1), np.repeat(be[..., None], dk, axis=-1),
                         np.repeat(be[..., None], dv, axis=-1), S0, dO, dST)
    g1 = oracle.gdr_bwd(q, k, v, la, be, S0, dO, dST)
    for n in ("dq", "dk", "dv", "dS0"):
        assert rel_err(g2[n], g1[n]) < 1e-11, n
    assert rel_err(g2["dlog_alpha"].sum(-1), g1["dlog_alpha"]) < 1e-11
    assert rel_err(g2["db"].sum(-1) + g2["dw"].sum(-1), g1["dbeta"]) < 1e-11
