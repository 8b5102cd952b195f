"""Small fp64 helpers shared by the oracle pin tests (numpy only)."""
import numpy as np


def rand_inputs(rng, B, T, H, dk, dv, s0=True, unit_k=True):
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk))
    if unit_k:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(B, T, H, dv))
    la = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(B, T, H))))
    be = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H))))
    S0 = rng.normal(scale=0.5, size=(B, H, dv, dk)) if s0 else None
    return q, k, v, la, be, S0


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))
