"""The affine segment map behind the sequence split, checked on the fp64
oracle (CPU only).

For one (b, h) the gated delta rule over a segment of tokens maps the
incoming state affinely: S_out = S_in M + N, where N is the segment's final
state from S_in = 0 and M = prod_t alpha_t (I - beta_t k_t k_t^T) in token
order (the chunkwise form's product of (gamma_C I - W^T K) factors, Gated
DeltaNet review, section 3.7).  The readout is affine too:
o_t = S_t q_t = S_in (M_<=t q_t) + o_t(S_in = 0).  Running the same rule with
v = 0 and S0 = I (dv = dk) yields S_T = M and outputs q~_t = M_<=t q_t, so a
segment needs two forward passes, an exchange of (M, N) and a small
correction o += S_in q~.  These tests compose those pieces, computed by the
oracle, and compare with one oracle pass over the whole sequence."""
import numpy as np
import pytest

import oracle
import synth


def segment_pieces(q, k, v, la, be):
    """(o0, N) with S_in = 0, and (q~, M) with v = 0, S_in = I."""
    B, T, H, dk = q.shape
    o0, N = oracle.gdr_fwd(q, k, v, la, be, None)
    eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
    qt, M = oracle.gdr_fwd(q, k, np.zeros_like(q), la, be, eye)
    return o0, N, qt, M


def compose(pieces, S0):
    """Sequential combine and the per-segment output correction."""
    S = S0.copy()
    outs = []
    for o0, N, qt, M in pieces:
        outs.append(o0 + np.einsum("bhij,bthj->bthi", S, qt))
        S = np.einsum("bhij,bhjk->bhik", S, M) + N
    return np.concatenate(outs, axis=1), S


@pytest.mark.parametrize("cuts", [[37], [64, 128], [1, 2, 3], [50, 51, 150]])
@pytest.mark.parametrize("dv", [8, 12])
def test_segments_compose_to_one_pass(cuts, dv):
    x = synth.gdr_inputs(2, 200, 2, 8, dv, "f32", seed=len(cuts) + dv, s0_std=0.5)
    x = {n: (t.double().numpy() if t is not None else None) for n, t in x.items()}
    q, k, v, la, be, S0 = (x[n] for n in ("q", "k", "v", "log_alpha", "beta", "S0"))
    o_ref, S_ref = oracle.gdr_fwd(q, k, v, la, be, S0)
    bounds = [0] + cuts + [q.shape[1]]
    pieces = [segment_pieces(q[:, a:b], k[:, a:b], v[:, a:b], la[:, a:b], be[:, a:b])
              for a, b in zip(bounds[:-1], bounds[1:])]
    o, S = compose(pieces, S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-10, atol=1e-12)


def test_transition_of_one_token_is_the_erase_factor():
    # one token: M = alpha (I - beta k k^T), q~ = M q
    rng = np.random.default_rng(3)
    dk = 6
    k = rng.standard_normal((1, 1, 1, dk))
    q = rng.standard_normal((1, 1, 1, dk))
    la = np.array([[[-0.3]]])
    be = np.array([[[0.7]]])
    _, _, qt, M = segment_pieces(q, k, np.zeros((1, 1, 1, 3)), la, be)
    kk = k[0, 0, 0]
    expect = np.exp(-0.3) * (np.eye(dk) - 0.7 * np.outer(kk, kk))
    np.testing.assert_allclose(M[0, 0], expect, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(qt[0, 0, 0], expect @ q[0, 0, 0], rtol=1e-14, atol=1e-15)
