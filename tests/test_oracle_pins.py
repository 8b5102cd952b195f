"""Pins of the fp64 oracle's forward and decode step to what the pages and
the mathematics fix (CPU only).

Each test checks the oracle against something other than itself:
  * a hand-worked example (tests/golden/gdr_worked_example.txt);
  * exact rational arithmetic on the literal product form of the rule;
  * the two written forms of the delta rule (product form vs error-correcting
    form, Gated DeltaNet review meaningful96.github.io/nr/GDN, section 3.3,
    derived as one SGD step in section 3.5) with the gate of section 3.4;
  * the write-then-read invariant for unit keys;
  * the readout timing o_t = S_t q_t (section 1);
  * closed forms for beta = 0 (pure decay, section 3.2 limit) and
    alpha = 1 (DeltaNet, section 3.3);
  * exact retrieval with orthonormal keys (section 2, "orthogonal key-value
    pairs");
  * explicit products of the transition matrices alpha_t (I - beta_t k k^T)
    (sections 3.3-3.4, generalised Householder transition).
A mistake such as a dropped alpha, a sign flip in the delta, a transposed
state or a readout before the update fails at least one of them.  dk != dv
throughout so that a transposed state cannot pass.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from pins_common import rand_inputs, rel_err


def _literal_product_form(q, k, v, la, be, S0):
    """S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T with
    dense matrices, o_t = S_t q_t (section 3.4 as printed)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    I = np.eye(dk)
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            for t in range(T):
                kk = k[b, t, h]
                a = math.exp(la[b, t, h])
                bt = be[b, t, h]
                S = S @ (a * (I - bt * np.outer(kk, kk))) + bt * np.outer(v[b, t, h], kk)
                o[b, t, h] = S @ q[b, t, h]
            ST[b, h] = S
    return o, ST


def test_worked_example(golden):
    g = golden("gdr_worked_example.txt")
    dk, dv = int(g["dk"][0]), int(g["dv"][0])
    T = len(g["alpha"])
    q = np.array(g["q"]).reshape(1, T, 1, dk)
    k = np.array(g["k"]).reshape(1, T, 1, dk)
    v = np.array(g["v"]).reshape(1, T, 1, dv)
    la = np.log(np.array(g["alpha"])).reshape(1, T, 1)
    be = np.array(g["beta"]).reshape(1, T, 1)
    S0 = np.array(g["S0"]).reshape(1, 1, dv, dk)
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    np.testing.assert_allclose(o.reshape(-1), g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(ST.reshape(-1), g["S_T"], rtol=0, atol=1e-14)


def test_exact_rational_arithmetic():
    """Exact Fractions through the literal product form vs the oracle."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 1, 4, 1, 3, 2
    # dyadic inputs are exact in binary floating point
    q = rng.integers(-8, 9, size=(B, T, H, dk)) / 8.0
    k = rng.integers(-8, 9, size=(B, T, H, dk)) / 8.0
    v = rng.integers(-8, 9, size=(B, T, H, dv)) / 4.0
    be = rng.integers(1, 16, size=(B, T, H)) / 16.0
    la = -rng.uniform(0.05, 1.0, size=(B, T, H))
    S0 = rng.integers(-4, 5, size=(B, H, dv, dk)) / 4.0
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)

    Fr = Fraction
    S = [[Fr(S0[0, 0, i, j]) for j in range(dk)] for i in range(dv)]
    o_ex = []
    for t in range(T):
        a = Fr(math.exp(la[0, t, 0]))
        bt = Fr(be[0, t, 0])
        kk = [Fr(x) for x in k[0, t, 0]]
        M = [[a * ((1 if i == j else 0) - bt * kk[i] * kk[j]) for j in range(dk)] for i in range(dk)]
        S = [[sum(S[i][m] * M[m][j] for m in range(dk)) + bt * Fr(v[0, t, 0, i]) * kk[j]
              for j in range(dk)] for i in range(dv)]
        o_ex.append([sum(S[i][j] * Fr(q[0, t, 0, j]) for j in range(dk)) for i in range(dv)])
    o_ex = np.array([[float(x) for x in row] for row in o_ex])
    S_ex = np.array([[float(x) for x in row] for row in S])
    np.testing.assert_allclose(o[0, :, 0], o_ex, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(ST[0, 0], S_ex, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("unit_k", [True, False])
def test_two_written_forms(unit_k):
    rng = np.random.default_rng(1)
    q, k, v, la, be, S0 = rand_inputs(rng, 2, 23, 3, 5, 3, unit_k=unit_k)
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    o2, ST2 = _literal_product_form(q, k, v, la, be, S0)
    assert rel_err(o, o2) < 1e-12
    assert rel_err(ST, ST2) < 1e-12


def test_write_then_read_invariant():
    """For unit k_t: S_t k_t = alpha_t (1 - beta_t) S_{t-1} k_t + beta_t v_t."""
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 1, 9, 2, 6, 4
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    prev = S0.copy()
    for t in range(1, T + 1):
        _, St = oracle.gdr_fwd(q[:, :t], k[:, :t], v[:, :t], la[:, :t], be[:, :t], S0)
        for h in range(H):
            kk = k[0, t - 1, h]
            a, bt = math.exp(la[0, t - 1, h]), be[0, t - 1, h]
            lhs = St[0, h] @ kk
            rhs = a * (1 - bt) * (prev[0, h] @ kk) + bt * v[0, t - 1, h]
            np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-13)
        prev = St


def test_beta_one_exact_write_then_read_and_readout_timing():
    """beta = 1, unit k: S_t k_t = v_t for any alpha; with q_t = k_t the
    readout (taken AFTER the update) returns v_t exactly."""
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 2, 12, 2, 7, 5
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    be[:] = 1.0
    o, _ = oracle.gdr_fwd(k, k, v, la, be, S0)
    np.testing.assert_allclose(o, v, rtol=1e-12, atol=1e-12)


def test_beta_zero_pure_decay():
    """beta = 0: S_t = (prod_{s<=t} alpha_s) S0 and o_t = S_t q_t."""
    rng = np.random.default_rng(4)
    B, T, H, dk, dv = 2, 15, 2, 6, 4
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    be[:] = 0.0
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    g = np.cumsum(la, axis=1)  # [B,T,H]
    exp_S = np.exp(g[:, -1])[:, :, None, None] * S0
    exp_o = np.exp(g)[..., None] * np.einsum("bhij,bthj->bthi", S0, q)
    assert rel_err(ST, exp_S) < 1e-13
    assert rel_err(o, exp_o) < 1e-13


def test_alpha_one_is_deltanet():
    """alpha = 1 gives DeltaNet, S_t = S_{t-1} + beta (v - S_{t-1} k) k^T."""
    rng = np.random.default_rng(5)
    B, T, H, dk, dv = 1, 20, 2, 6, 3
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la[:] = 0.0
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kk = k[0, t, h]
            S = S + be[0, t, h] * np.outer(v[0, t, h] - S @ kk, kk)
            np.testing.assert_allclose(o[0, t, h], S @ q[0, t, h], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ST[0, h], S, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T", [1, 7, 16])
def test_orthonormal_retrieval(T):
    """T <= dk orthonormal keys, alpha = beta = 1, S0 = 0: every stored value
    is retrieved exactly and S_T = sum_i v_i k_i^T."""
    rng = np.random.default_rng(6 + T)
    dk, dv = 16, 5
    Qm, _ = np.linalg.qr(rng.normal(size=(dk, dk)))
    keys = Qm.T[:T]                          # orthonormal rows
    k = keys.reshape(1, T, 1, dk)
    v = rng.normal(size=(1, T, 1, dv))
    q = rng.normal(size=(1, T, 1, dk))
    la = np.zeros((1, T, 1))
    be = np.ones((1, T, 1))
    _, ST = oracle.gdr_fwd(q, k, v, la, be, None)
    S = ST[0, 0]
    for i in range(T):
        np.testing.assert_allclose(S @ keys[i], v[0, i, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, v[0, :, 0].T @ keys, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T", [1, 3, 8])
def test_transition_products(T):
    """S_T = S0 prod_t A_t + sum_t beta_t v_t k_t^T prod_{s>t} A_s with
    A_t = alpha_t (I - beta_t k_t k_t^T), as explicit dense products."""
    rng = np.random.default_rng(20 + T)
    B, H, dk, dv = 1, 2, 5, 4
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv, unit_k=False)
    _, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    for h in range(H):
        A = [math.exp(la[0, t, h]) * (np.eye(dk) - be[0, t, h] * np.outer(k[0, t, h], k[0, t, h]))
             for t in range(T)]

        def prod(lo):
            M = np.eye(dk)
            for s in range(lo, T):
                M = M @ A[s]
            return M

        S = S0[0, h] @ prod(0)
        for t in range(T):
            S = S + be[0, t, h] * np.outer(v[0, t, h], k[0, t, h]) @ prod(t + 1)
        np.testing.assert_allclose(ST[0, h], S, rtol=1e-11, atol=1e-12)


def test_step_sequence_equals_forward():
    """T decode steps reproduce the forward's outputs and final state."""
    rng = np.random.default_rng(7)
    B, T, H, dk, dv = 3, 11, 2, 6, 5
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    S = S0.copy()
    for t in range(T):
        ot, S = oracle.gdr_step(q[:, t], k[:, t], v[:, t], la[:, t], be[:, t], S)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S, ST, rtol=1e-13, atol=1e-14)


def test_zero_length_and_null_state():
    rng = np.random.default_rng(8)
    q, k, v, la, be, _ = rand_inputs(rng, 1, 5, 1, 4, 3)
    o, ST = oracle.gdr_fwd(q, k, v, la, be, None)
    o2, ST2 = oracle.gdr_fwd(q, k, v, la, be, np.zeros((1, 1, 3, 4)))
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(ST, ST2)
