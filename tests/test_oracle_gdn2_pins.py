"""Pins of the oracle's Gated DeltaNet-2 forward (CPU only, fp64).

Source: "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
(agihunt.info/papers/2605.22791), the Gated Delta Rule-2 paragraph: the two
channel gates collapse to one scalar -> KDA; the decay collapsing to a scalar
as well -> Gated DeltaNet.  Checks:
  * the hand-worked example in tests/golden/gdr2_worked_example.txt;
  * collapse b = w = beta*1, scalar alpha  ==  the gated delta rule oracle;
  * vector alpha with b = w = beta*1  ==  an independent KDA-form loop
    S_t = (S_{t-1} Diag(alpha_t)) (I - beta_t k k^T) + beta_t v k^T;
  * b = 0 (no erase) closed form
    S_T = S0 Diag(prod alpha) + sum_i (w_i*v_i)(k_i * prod_{s>i} alpha_s)^T;
  * explicit transition products for T <= 8.
"""
import math

import numpy as np
import pytest

import oracle
from pins_common import rand_inputs, rel_err


def _gates(rng, B, T, H, dk, dv):
    la = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(B, T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H, dk))))
    w = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H, dv))))
    return la, b, w


def test_worked_example(golden):
    g = golden("gdr2_worked_example.txt")
    dk, dv = int(g["dk"][0]), int(g["dv"][0])
    T = len(g["alpha"]) // dk
    sh = lambda key, d: np.array(g[key]).reshape(1, T, 1, d)
    o, ST = oracle.gdr2_fwd(sh("q", dk), sh("k", dk), sh("v", dv), np.log(sh("alpha", dk)),
                            sh("b", dk), sh("w", dv), np.array(g["S0"]).reshape(1, 1, dv, dk))
    np.testing.assert_allclose(o.reshape(-1), g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(ST.reshape(-1), g["S_T"], rtol=0, atol=1e-14)


def test_collapse_to_gated_delta_rule():
    rng = np.random.default_rng(40)
    B, T, H, dk, dv = 2, 30, 2, 6, 4
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la_c = np.repeat(la[..., None], dk, axis=-1)
    b = np.repeat(be[..., None], dk, axis=-1)
    w = np.repeat(be[..., None], dv, axis=-1)
    o2, ST2 = oracle.gdr2_fwd(q, k, v, la_c, b, w, S0)
    o1, ST1 = oracle.gdr_fwd(q, k, v, la, be, S0)
    assert rel_err(o2, o1) < 1e-12
    assert rel_err(ST2, ST1) < 1e-12


def test_collapse_to_kda_form():
    rng = np.random.default_rng(41)
    B, T, H, dk, dv = 1, 17, 2, 5, 3
    q, k, v, _, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la, _, _ = _gates(rng, B, T, H, dk, dv)
    b = np.repeat(be[..., None], dk, axis=-1)
    w = np.repeat(be[..., None], dv, axis=-1)
    o, ST = oracle.gdr2_fwd(q, k, v, la, b, w, S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kk = k[0, t, h]
            bt = be[0, t, h]
            S = (S @ np.diag(np.exp(la[0, t, h]))) @ (np.eye(dk) - bt * np.outer(kk, kk)) \
                + bt * np.outer(v[0, t, h], kk)
            np.testing.assert_allclose(o[0, t, h], S @ q[0, t, h], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ST[0, h], S, rtol=1e-12, atol=1e-13)


def test_no_erase_closed_form():
    rng = np.random.default_rng(42)
    B, T, H, dk, dv = 1, 13, 2, 5, 4
    q, k, v, _, _, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la, b, w = _gates(rng, B, T, H, dk, dv)
    b[:] = 0.0
    _, ST = oracle.gdr2_fwd(q, k, v, la, b, w, S0)
    G = np.cumsum(la, axis=1)  # [B,T,H,dk]
    for h in range(H):
        S = S0[0, h] * np.exp(G[0, -1, h])[None, :]
        for i in range(T):
            S = S + np.outer(w[0, i, h] * v[0, i, h], k[0, i, h] * np.exp(G[0, -1, h] - G[0, i, h]))
        np.testing.assert_allclose(ST[0, h], S, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T", [1, 4, 8])
def test_transition_products(T):
    """S_t = S_{t-1} Diag(alpha_t)(I - (b_t*k_t) k_t^T) + (w_t*v_t) k_t^T,
    unrolled into explicit dense products."""
    rng = np.random.default_rng(50 + T)
    B, H, dk, dv = 1, 1, 5, 3
    q, k, v, _, _, S0 = rand_inputs(rng, B, T, H, dk, dv, unit_k=False)
    la, b, w = _gates(rng, B, T, H, dk, dv)
    _, ST = oracle.gdr2_fwd(q, k, v, la, b, w, S0)
    A = [np.diag(np.exp(la[0, t, 0])) @ (np.eye(dk) - np.outer(b[0, t, 0] * k[0, t, 0], k[0, t, 0]))
         for t in range(T)]

    def prod(lo):
        M = np.eye(dk)
        for s in range(lo, T):
            M = M @ A[s]
        return M

    S = S0[0, 0] @ prod(0)
    for t in range(T):
        S = S + np.outer(w[0, t, 0] * v[0, t, 0], k[0, t, 0]) @ prod(t + 1)
    np.testing.assert_allclose(ST[0, 0], S, rtol=1e-11, atol=1e-12)


def test_erase_gate_two_is_a_householder_reflection():
    """Negative-eigenvalue range (erase gate b in [0, 2], the Gated DeltaNet-2
    page's remark on extending the erase gate): with unit keys, no decay and
    b = 2 on every channel, the erase factor I - 2 k k^T is a reflection, so
    each step gives S_t k_t = -S_{t-1} k_t + w_t*v_t exactly (fp64)."""
    rng = np.random.default_rng(44)
    B, T, H, dk, dv = 1, 12, 1, 6, 4
    k = rng.normal(size=(B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = rng.normal(size=(B, T, H, dk))
    v = rng.normal(size=(B, T, H, dv))
    w = rng.uniform(0.1, 1.0, size=(B, T, H, dv))
    b = np.full((B, T, H, dk), 2.0)
    la = np.zeros((B, T, H, dk))
    S = rng.normal(size=(B, H, dv, dk))
    for t in range(T):
        sl = lambda x: x[:, t:t + 1]
        _, S_next = oracle.gdr2_fwd(sl(q), sl(k), sl(v), sl(la), sl(b), sl(w), S)
        kt = k[0, t, 0]
        lhs = S_next[0, 0] @ kt
        rhs = -(S[0, 0] @ kt) + w[0, t, 0] * v[0, t, 0]
        assert np.abs(lhs - rhs).max() < 1e-12
        # the reflection preserves the part of the state orthogonal to k
        u = rng.normal(size=dk)
        u -= (u @ kt) * kt
        assert np.abs(S_next[0, 0] @ u - S[0, 0] @ u).max() < 1e-12
        S = S_next
