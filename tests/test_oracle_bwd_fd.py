"""Pin of the oracle's hand-derived reverse mode to central finite
differences of the oracle's forward (CPU only, fp64).

Loss L = <dO, o> + <dS_T, S_T>.  Every input element (q, k, v, log alpha,
beta, S0) is perturbed by +-h and (L(x+h) - L(x-h)) / 2h is compared with the
analytic gradient.  A dropped term or a wrong sign in any of the six
gradients fails here.  The T = 70 case crosses the oracle's 64-token
recomputation block boundary.
"""
import numpy as np
import pytest

import oracle
from pins_common import rand_inputs


def _loss(args, dO, dST):
    o, ST = oracle.gdr_fwd(*args)
    return float(np.sum(o * dO) + np.sum(ST * dST))


@pytest.mark.parametrize("T,dk,dv,sample", [(9, 4, 3, None), (70, 3, 2, 60)])
def test_bwd_matches_finite_differences(T, dk, dv, sample):
    rng = np.random.default_rng(100 + T)
    B, H = 1, 2
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    dO = rng.normal(size=(B, T, H, dv))
    dST = rng.normal(size=(B, H, dv, dk))
    g = oracle.gdr_bwd(q, k, v, la, be, S0, dO, dST)
    names = ["q", "k", "v", "log_alpha", "beta", "S0"]
    grads = [g["dq"], g["dk"], g["dv"], g["dlog_alpha"], g["dbeta"], g["dS0"]]
    args = [q, k, v, la, be, S0]
    h = 1e-6
    for ai, (name, grad) in enumerate(zip(names, grads)):
        x = args[ai]
        idx = np.arange(x.size)
        if sample is not None and x.size > sample:
            idx = rng.choice(x.size, size=sample, replace=False)
        for flat in idx:
            pos = np.unravel_index(flat, x.shape)
            old = x[pos]
            x[pos] = old + h
            lp = _loss(args, dO, dST)
            x[pos] = old - h
            lm = _loss(args, dO, dST)
            x[pos] = old
            fd = (lp - lm) / (2 * h)
            an = grad[pos]
            assert abs(fd - an) <= 2e-6 * (1.0 + abs(an)), (name, pos, fd, an)


def test_bwd_closed_form_pure_decay():
    """beta = 0, dO = 0: dS0 = (prod alpha) dS_T and
    dlog_alpha_t = <dS_T, S_T> for every t (S_T = exp(sum log alpha) S0)."""
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 1, 6, 1, 4, 3
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    be[:] = 0.0
    dO = np.zeros((B, T, H, dv))
    dST = rng.normal(size=(B, H, dv, dk))
    g = oracle.gdr_bwd(q, k, v, la, be, S0, dO, dST)
    decay = np.exp(la.sum())
    np.testing.assert_allclose(g["dS0"], decay * dST, rtol=1e-13)
    np.testing.assert_allclose(g["dlog_alpha"], np.full((B, T, H), decay * np.sum(dST * S0)),
                               rtol=1e-12)
    np.testing.assert_allclose(g["dq"], 0.0, atol=0)
