"""Pin of the chunkwise (UT transform / WY) reading that the CUDA kernels
implement, against the sequential oracle (CPU only, fp64).

The chunkwise equations are printed in the Gated DeltaNet review
(meaningful96.github.io/nr/GDN), section 3.7, partly garbled: the arrow
decorations are undefined, W is never defined and the intra-chunk mask has
lost its decay.  The reading taken (derived by substituting the ansatz
S_r = gamma_r S + sum_{i<=r} (gamma_r/gamma_i) u_i k_i^T into the rule of
section 3.4) is, per chunk of C tokens with g_r = sum_{s<=r} log alpha_s,
gamma_r = exp(g_r):

    A     = strictLower(diag(beta) (Gamma * K K^T)),  Gamma_ri = gamma_r/gamma_i
    T     = (I + A)^-1
    U^g   = T diag(beta) V
    W     = T diag(beta*gamma) K
    U     = U^g - W S^T
    O     = diag(gamma) Q S^T + (Q K^T * L) U,        L_ri = gamma_r/gamma_i, i <= r
    S'    = gamma_C S + U^T diag(gamma_C/gamma) K

and for Gated DeltaNet-2 ("Gated DeltaNet-2: Decoupling Erase and Write in
Linear Attention", agihunt.info/papers/2605.22791: the channel decay is
absorbed into an asymmetric rank-1 erase factor, WY triangular solve at
chunk 64), with E = exp(per-channel cumulative log alpha):

    A  = strictLower((K*B*E)(K/E)^T),  U = (I + A)^-1 ((W*V) - (K*B*E) S^T)
    O  = (Q*E) S^T + (((Q*E)(K/E)^T) * M_incl) U
    S' = S Diag(E_C) + U^T (K * E_C/E)

If this reading were wrong (a missing decay on the mask, gamma on the wrong
side of T, a wrong transpose) the comparison below would fail by O(1).
The result must not depend on C; C = 1 is the recurrence itself.
"""
import numpy as np
import pytest

import oracle
from pins_common import rand_inputs, rel_err


def chunkwise_gdr(q, k, v, la, be, S0, C):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, min(c0 + C, T))
                Q, K, V = q[b, sl, h], k[b, sl, h], v[b, sl, h]
                beta = be[b, sl, h]
                g = np.cumsum(la[b, sl, h])
                n = len(g)
                ratio = np.exp(g[:, None] - g[None, :])
                strict = np.tril(np.ones((n, n)), -1)
                incl = np.tril(np.ones((n, n)))
                A = strict * (beta[:, None] * ratio * (K @ K.T))
                Tm = np.linalg.inv(np.eye(n) + A)
                Ug = Tm @ (beta[:, None] * V)
                W = Tm @ ((beta * np.exp(g))[:, None] * K)
                U = Ug - W @ S.T
                o[b, sl, h] = np.exp(g)[:, None] * (Q @ S.T) + ((Q @ K.T) * ratio * incl) @ U
                S = np.exp(g[-1]) * S + U.T @ (np.exp(g[-1] - g)[:, None] * K)
            ST[b, h] = S
    return o, ST


def chunkwise_gdr2(q, k, v, la, bg, wg, S0, C):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, min(c0 + C, T))
                Q, K, V = q[b, sl, h], k[b, sl, h], v[b, sl, h]
                G = np.cumsum(la[b, sl, h], axis=0)
                E = np.exp(G)
                n = G.shape[0]
                strict = np.tril(np.ones((n, n)), -1)
                incl = np.tril(np.ones((n, n)))
                KBE = K * bg[b, sl, h] * E
                A = strict * (KBE @ (K / E).T)
                Tm = np.linalg.inv(np.eye(n) + A)
                U = Tm @ (wg[b, sl, h] * V - KBE @ S.T)
                QE = Q * E
                o[b, sl, h] = QE @ S.T + ((QE @ (K / E).T) * incl) @ U
                S = S * E[-1][None, :] + U.T @ (K * np.exp(G[-1][None, :] - G))
            ST[b, h] = S
    return o, ST


@pytest.mark.parametrize("C", [1, 4, 64])
@pytest.mark.parametrize("T", [64, 100, 256])
def test_chunkwise_gdr_equals_recurrence(C, T):
    rng = np.random.default_rng(C * 1000 + T)
    q, k, v, la, be, S0 = rand_inputs(rng, 1, T, 2, 8, 6)
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    oc, STc = chunkwise_gdr(q, k, v, la, be, S0, C)
    assert rel_err(oc, o) < 1e-11
    assert rel_err(STc, ST) < 1e-11


@pytest.mark.parametrize("C", [1, 4, 64])
@pytest.mark.parametrize("T", [64, 100])
def test_chunkwise_gdr2_equals_recurrence(C, T):
    rng = np.random.default_rng(7 * C + T)
    q, k, v, _, _, S0 = rand_inputs(rng, 1, T, 2, 8, 6)
    la = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(1, T, 2, 8))))
    bg = 1.0 / (1.0 + np.exp(-rng.normal(size=(1, T, 2, 8))))
    wg = 1.0 / (1.0 + np.exp(-rng.normal(size=(1, T, 2, 6))))
    o, ST = oracle.gdr2_fwd(q, k, v, la, bg, wg, S0)
    oc, STc = chunkwise_gdr2(q, k, v, la, bg, wg, S0, C)
    assert rel_err(oc, o) < 1e-10
    assert rel_err(STc, ST) < 1e-10


def chunkwise_gdr_u_chain(q, k, v, la, be, S0, C):
    """The chunkwise forward with U carried chunk to chunk instead of formed
    from the freshly updated state.  With S_{n+1} = gamma_C S_n + U_n^T Kd_n
    (Kd = diag(gamma_C/gamma) K), U_{n+1} = U^g_{n+1} - W_{n+1} S_{n+1}^T
    expands to

        U_{n+1} = U^g_{n+1} - gamma_C W_{n+1} S_n^T - (W_{n+1} Kd_n^T) U_n,

    so U_{n+1} needs S_n (one step old) and U_n, and the state update leaves
    the chain from U_n to U_{n+1}.  Algebraically the same map; a state-pass
    kernel may take either form."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            prev = None  # (S_n, gamma_C, Kd, U) of the chunk before
            for c0 in range(0, T, C):
                sl = slice(c0, min(c0 + C, T))
                Q, K, V = q[b, sl, h], k[b, sl, h], v[b, sl, h]
                beta = be[b, sl, h]
                g = np.cumsum(la[b, sl, h])
                n = len(g)
                ratio = np.exp(g[:, None] - g[None, :])
                A = np.tril(np.ones((n, n)), -1) * (beta[:, None] * ratio * (K @ K.T))
                Tm = np.linalg.inv(np.eye(n) + A)
                Ug = Tm @ (beta[:, None] * V)
                W = Tm @ ((beta * np.exp(g))[:, None] * K)
                if prev is None:
                    U = Ug - W @ S.T
                else:
                    Sp, gCp, Kdp, Up = prev
                    U = Ug - gCp * (W @ Sp.T) - (W @ Kdp.T) @ Up
                o[b, sl, h] = np.exp(g)[:, None] * (Q @ S.T) + ((Q @ K.T) * ratio * np.tril(np.ones((n, n)))) @ U
                Kd = np.exp(g[-1] - g)[:, None] * K
                prev = (S, np.exp(g[-1]), Kd, U)
                S = np.exp(g[-1]) * S + U.T @ Kd
            ST[b, h] = S
    return o, ST


@pytest.mark.parametrize("C", [4, 64])
@pytest.mark.parametrize("T", [64, 200, 256])
def test_u_chain_form_equals_recurrence(C, T):
    rng = np.random.default_rng(3 * C + T)
    q, k, v, la, be, S0 = rand_inputs(rng, 1, T, 2, 8, 6)
    o, ST = oracle.gdr_fwd(q, k, v, la, be, S0)
    oc, STc = chunkwise_gdr_u_chain(q, k, v, la, be, S0, C)
    assert rel_err(oc, o) < 1e-10
    assert rel_err(STc, ST) < 1e-10


def test_u_chain_form_needs_the_decay_on_the_old_state():
    """Dropping gamma_C from the S_n term (a plausible slip when moving the
    state update off the chain) is off by O(1)."""
    rng = np.random.default_rng(5)
    q, k, v, la, be, S0 = rand_inputs(rng, 1, 128, 1, 8, 6)
    o, _ = oracle.gdr_fwd(q, k, v, la, be, S0)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    beta, g_all = be[0, :, 0], la[0, :, 0]
    S = S0[0, 0]
    parts = []
    for c0 in (0, 64):
        sl = slice(c0, c0 + 64)
        g = np.cumsum(g_all[sl])
        ratio = np.exp(g[:, None] - g[None, :])
        A = np.tril(np.ones((64, 64)), -1) * (beta[sl][:, None] * ratio * (K[sl] @ K[sl].T))
        Tm = np.linalg.inv(np.eye(64) + A)
        Ug = Tm @ (beta[sl][:, None] * V[sl])
        W = Tm @ ((beta[sl] * np.exp(g))[:, None] * K[sl])
        parts.append((g, ratio, Ug, W))
    g0, r0, Ug0, W0 = parts[0]
    U0 = Ug0 - W0 @ S.T
    Kd0 = np.exp(g0[-1] - g0)[:, None] * K[:64]
    S1 = np.exp(g0[-1]) * S + U0.T @ Kd0
    g1, r1, Ug1, W1 = parts[1]
    U1_bad = Ug1 - W1 @ S.T - (W1 @ Kd0.T) @ U0
    o1_bad = np.exp(g1)[:, None] * (Q[64:] @ S1.T) + ((Q[64:] @ K[64:].T) * r1 * np.tril(np.ones((64, 64)))) @ U1_bad
    assert rel_err(o1_bad, o[0, 64:, 0]) > 1e-3


def test_mask_without_decay_is_wrong():
    """The literal printed mask (no decay on the intra-chunk term) disagrees
    with the recurrence, which is why the decayed mask is the reading."""
    rng = np.random.default_rng(9)
    q, k, v, la, be, S0 = rand_inputs(rng, 1, 64, 1, 8, 6)
    o, _ = oracle.gdr_fwd(q, k, v, la, be, S0)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    beta = be[0, :, 0]
    g = np.cumsum(la[0, :, 0])
    n = 64
    ratio = np.exp(g[:, None] - g[None, :])
    A = np.tril(np.ones((n, n)), -1) * (beta[:, None] * ratio * (K @ K.T))
    Tm = np.linalg.inv(np.eye(n) + A)
    S = S0[0, 0]
    U = Tm @ (beta[:, None] * V) - Tm @ ((beta * np.exp(g))[:, None] * K) @ S.T
    o_bad = np.exp(g)[:, None] * (Q @ S.T) + ((Q @ K.T) * np.tril(np.ones((n, n)))) @ U
    assert rel_err(o_bad, o[0, :, 0]) > 1e-2


def chunkwise_gdr_bwd(q, k, v, la, be, S0, dO, dST, C=64):
    """Per-chunk reverse mode of the chunkwise reading above (the formulas
    the CUDA backward evaluates), fp64."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    g_all = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dla", la),
                                              ("dbe", be))}
    dS0 = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            # forward: chunk entry states
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            starts = []
            for c0 in range(0, T, C):
                starts.append(S.copy())
                sl = slice(c0, min(c0 + C, T))
                _, S = _chunk_fwd(q[b, sl, h], k[b, sl, h], v[b, sl, h], la[b, sl, h],
                                  be[b, sl, h], S)
            D = dST[b, h].copy() if dST is not None else np.zeros((dv, dk))
            for ci in reversed(range(len(starts))):
                c0 = ci * C
                sl = slice(c0, min(c0 + C, T))
                Q, K, V, dOc = q[b, sl, h], k[b, sl, h], v[b, sl, h], dO[b, sl, h]
                beta = be[b, sl, h]
                S = starts[ci]
                n = Q.shape[0]
                g = np.cumsum(la[b, sl, h])
                gam = np.exp(g)
                dec = np.exp(g[-1] - g)
                ratio = np.exp(g[:, None] - g[None, :])
                strict = np.tril(np.ones((n, n)), -1)
                incl = np.tril(np.ones((n, n)))
                G = strict * ratio * (K @ K.T)
                A = beta[:, None] * G
                P = incl * ratio * (Q @ K.T)
                X = K @ S.T
                Y = Q @ S.T
                R = beta[:, None] * (V - gam[:, None] * X)
                U = np.linalg.solve(np.eye(n) + A, R)
                dU = dec[:, None] * (K @ D.T) + P.T @ dOc
                dP = incl * (dOc @ U.T)
                dR = np.linalg.solve((np.eye(n) + A).T, dU)
                dA = -strict * (dR @ U.T)
                dPL = dP * incl * ratio
                dKK = dA * beta[:, None] * ratio * strict
                UD = dec[:, None] * (U @ D)
                dQ = gam[:, None] * (dOc @ S) + dPL @ K
                dK = dPL.T @ Q + dKK @ K + dKK.T @ K + UD - (beta * gam)[:, None] * (dR @ S)
                db = np.sum(dR * (V - gam[:, None] * X), 1) + np.sum(dA * G, 1)
                E, F = dP * P, dA * A
                z = np.sum(UD * K, 1)
                dg = (gam * np.sum(dOc * Y, 1) - beta * gam * np.sum(dR * X, 1) - z
                      + E.sum(1) - E.sum(0) + F.sum(1) - F.sum(0))
                dg[-1] += gam[-1] * np.sum(D * S) + z.sum()
                g_all["dq"][b, sl, h] = dQ
                g_all["dk"][b, sl, h] = dK
                g_all["dv"][b, sl, h] = beta[:, None] * dR
                g_all["dbe"][b, sl, h] = db
                g_all["dla"][b, sl, h] = np.cumsum(dg[::-1])[::-1]
                D = gam[-1] * D + dOc.T @ (gam[:, None] * Q) - dR.T @ ((beta * gam)[:, None] * K)
            dS0[b, h] = D
    return dict(dq=g_all["dq"], dk=g_all["dk"], dv=g_all["dv"], dlog_alpha=g_all["dla"],
                dbeta=g_all["dbe"], dS0=dS0)


def _chunk_fwd(Q, K, V, la, beta, S):
    g = np.cumsum(la)
    n = len(g)
    ratio = np.exp(g[:, None] - g[None, :])
    A = np.tril(np.ones((n, n)), -1) * (beta[:, None] * ratio * (K @ K.T))
    U = np.linalg.solve(np.eye(n) + A, beta[:, None] * (V - np.exp(g)[:, None] * (K @ S.T)))
    O = np.exp(g)[:, None] * (Q @ S.T) + ((Q @ K.T) * ratio * np.tril(np.ones((n, n)))) @ U
    return O, np.exp(g[-1]) * S + U.T @ (np.exp(g[-1] - g)[:, None] * K)


@pytest.mark.parametrize("T,C", [(64, 64), (100, 64), (150, 16), (37, 8)])
def test_chunkwise_backward_equals_oracle_reverse_mode(T, C):
    rng = np.random.default_rng(T + C)
    q, k, v, la, be, S0 = rand_inputs(rng, 1, T, 2, 8, 6)
    dO = rng.normal(size=v.shape)
    dST = rng.normal(size=(1, 2, 6, 8))
    ref = oracle.gdr_bwd(q, k, v, la, be, S0, dO, dST)
    got = chunkwise_gdr_bwd(q, k, v, la, be, S0, dO, dST, C)
    for name in ref:
        assert rel_err(got[name], ref[name]) < 1e-10, name


def chunkwise_gdr2_bwd(q, k, v, la, bg, wg, S0, dO, dST, C=64, scaled_d=True):
    """Per-chunk reverse mode of the Gated DeltaNet-2 chunk form (the formulas
    the tensor-core GDN-2 backward evaluates), fp64.  Per chunk, with S the
    entry state, D = dL/dS' the exit-state gradient and
    KBE = K*B*E, QE = Q*E, KiE = K/E, Kt = K*exp(G_C - G) = KiE Diag(E_C):
        dU = Kt D^T + P^T dO,   dR = T^T dU,
        dA = -strictLower(dR U^T),   dP = inclLower(dO U^T),
        dKBE = -dR S + dA KiE,   dQE = dO S + dP KiE,
        dKiE = dA^T KBE + dP^T QE + (U D) Diag(E_C),
        dE_C = colsum(S*D) + colsum((U D)*KiE),
        D_prev = D Diag(E_C) + dO^T QE - dR^T KBE,
    then dk = dKBE*B*E + dKiE/E, db = dKBE*K*E, dq = dQE*E, dv = W*dR,
    dw = V*dR, dG = dKBE*KBE + dQE*QE - dKiE*KiE (+ E_C dE_C on the last
    token) and dlog alpha = the in-chunk suffix sums of dG.  scaled_d uses
    D' = D Diag(E_C) with KiE, the form the per-chunk kernel multiplies:
    Kt D^T = KiE D'^T and (U D) Diag(E_C) = U D'."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dlog_alpha", la),
                                            ("db", bg), ("dw", wg))}
    out["dS0"] = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            starts = []
            for c0 in range(0, T, C):
                starts.append(S.copy())
                sl = slice(c0, min(c0 + C, T))
                Q, K, V = q[b, sl, h], k[b, sl, h], v[b, sl, h]
                G = np.cumsum(la[b, sl, h], axis=0)
                E = np.exp(G)
                n = G.shape[0]
                KBE = K * bg[b, sl, h] * E
                A = np.tril(np.ones((n, n)), -1) * (KBE @ (K / E).T)
                U = np.linalg.inv(np.eye(n) + A) @ (wg[b, sl, h] * V - KBE @ S.T)
                S = S * E[-1][None, :] + U.T @ (K * np.exp(G[-1][None, :] - G))
            D = dST[b, h].copy() if dST is not None else np.zeros((dv, dk))
            for ci in reversed(range(len(starts))):
                sl = slice(ci * C, min(ci * C + C, T))
                Q, K, V, dOc = q[b, sl, h], k[b, sl, h], v[b, sl, h], dO[b, sl, h]
                Bg, Wg = bg[b, sl, h], wg[b, sl, h]
                S = starts[ci]
                G = np.cumsum(la[b, sl, h], axis=0)
                E = np.exp(G)
                EC = E[-1]
                n = G.shape[0]
                strict = np.tril(np.ones((n, n)), -1)
                incl = np.tril(np.ones((n, n)))
                KBE, QE, KiE = K * Bg * E, Q * E, K / E
                Kt = K * np.exp(G[-1][None, :] - G)
                A = strict * (KBE @ KiE.T)
                P = incl * (QE @ KiE.T)
                Tm = np.linalg.inv(np.eye(n) + A)
                R = Wg * V - KBE @ S.T
                U = Tm @ R
                if scaled_d:
                    Dp = D * EC[None, :]
                    dU = KiE @ Dp.T + P.T @ dOc
                    UDs = U @ Dp
                else:
                    dU = Kt @ D.T + P.T @ dOc
                    UDs = (U @ D) * EC[None, :]
                dR = Tm.T @ dU
                dA = -strict * (dR @ U.T)
                dP = incl * (dOc @ U.T)
                dKBE = -dR @ S + dA @ KiE
                dQE = dOc @ S + dP @ KiE
                dKiE = dA.T @ KBE + dP.T @ QE + UDs
                dEC = np.sum(S * D, 0) + np.sum(UDs * KiE, 0) / EC
                dG = dKBE * KBE + dQE * QE - dKiE * KiE
                dG[-1] += EC * dEC
                out["dq"][b, sl, h] = dQE * E
                out["dk"][b, sl, h] = dKBE * Bg * E + dKiE / E
                out["db"][b, sl, h] = dKBE * K * E
                out["dv"][b, sl, h] = Wg * dR
                out["dw"][b, sl, h] = V * dR
                out["dlog_alpha"][b, sl, h] = np.cumsum(dG[::-1], axis=0)[::-1]
                D = D * EC[None, :] + dOc.T @ QE - dR.T @ KBE
            out["dS0"][b, h] = D
    return out


def _gdr2_bwd_inputs(rng, T):
    q, k, v, _, _, S0 = rand_inputs(rng, 1, T, 2, 8, 6)
    la = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(1, T, 2, 8))))
    bg = rng.uniform(0.0, 2.0, size=(1, T, 2, 8))
    wg = rng.uniform(0.0, 1.0, size=(1, T, 2, 6))
    dO = rng.normal(size=(1, T, 2, 6))
    dST = rng.normal(size=(1, 2, 6, 8))
    return q, k, v, la, bg, wg, S0, dO, dST


@pytest.mark.parametrize("scaled_d", [False, True])
@pytest.mark.parametrize("T,C", [(64, 64), (150, 64), (100, 16)])
def test_chunkwise_gdr2_backward_equals_oracle_reverse_mode(T, C, scaled_d):
    rng = np.random.default_rng(11 * T + C)
    q, k, v, la, bg, wg, S0, dO, dST = _gdr2_bwd_inputs(rng, T)
    ref = oracle.gdr2_bwd(q, k, v, la, bg, wg, S0, dO, dST)
    got = chunkwise_gdr2_bwd(q, k, v, la, bg, wg, S0, dO, dST, C=C, scaled_d=scaled_d)
    for name in ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"):
        assert rel_err(got[name], ref[name]) < 1e-9, name
