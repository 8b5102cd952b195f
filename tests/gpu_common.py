"""Helpers for the GPU parity tests: move seeded inputs to the device and
compare with the oracle under the stated tolerances."""
import numpy as np
import torch

# Tolerances of the parity contract: max|d o| / max|o_ref| (per dtype of the
# inputs) and the relative Frobenius error of the final state.
TOL_O = {"f32": 1e-4, "bf16": 2e-2}
TOL_S = 1e-2
# Gradients (the pages state none): max|d| / max|ref| per tensor, 2e-2 for
# bf16 inputs and 1e-4 for fp32 inputs; dS0 relative Frobenius 1e-2.
TOL_G = {"f32": 1e-4, "bf16": 2e-2}


def dev(x):
    return None if x is None else x.cuda().contiguous()


def np64(x):
    return None if x is None else x.detach().double().cpu().numpy()


def max_rel(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(a - ref)) / max(np.max(np.abs(ref)), 1e-30))


def fro_rel(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-30))


def dtype_name(t: torch.Tensor) -> str:
    return "f32" if t.dtype == torch.float32 else "bf16"
