"""Seeded synthetic inputs for the gated delta rule.

This module is shared by the CUDA path's tests/bench and by the oracle's
tests; it contains none of the recurrence's arithmetic, only the input
distributions:

* q, k ~ N(0,1), then L2-normalised per (b, t, h) in fp32 (x / ||x||_2, no
  epsilon), then cast to the storage dtype -- the Gated DeltaNet block
  normalises q and k before the token mixer (Gated DeltaNet review,
  meaningful96.github.io/nr/GDN, section 3.8).
* v ~ N(0,1), cast to the storage dtype.
* log alpha = -softplus(x), x ~ N(-2, 1), fp32  (alpha in (0,1)).
* beta = sigmoid(N(0,1)), fp32                  (beta in (0,1)).
* S0 ~ N(0, 0.02^2) fp32 (0.02 is a standard deviation) or all zeros.
* dO ~ N(0,1) in the storage dtype.
* Gated DeltaNet-2: log alpha per key channel -softplus(N(-2,1)), erase gate
  b = sigmoid(N(0,1)) per key channel, write gate w = sigmoid(N(0,1)) per
  value channel, all fp32.

* Block prologue/epilogue (the pre- and post-processing of the Gated
  DeltaNet block): projected inputs xq, xk, xv ~ N(0,1) in the storage dtype;
  ShortConv taps ~ U(-1/sqrt(K), 1/sqrt(K)) fp32 (the usual fan-in bound of a
  depthwise convolution), biases ~ U(-1/sqrt(K), 1/sqrt(K)) fp32 or none, conv
  state ~ N(0,1) in the storage dtype or none; recurrent output o ~ N(0, 0.1^2)
  and gate projection g ~ N(0,1) in the storage dtype, norm weight
  1 + N(0, 0.1^2) fp32.  Draw order: xq, xk, xv, wq, wk, wv, bq, bk, bv,
  state; and o, g, weight.

Draw order from one torch CPU Generator seeded with `seed`:
q, k, v, x_alpha, x_beta, S0, dO for the scalar-gate rule;
q, k, v, x_alpha (per channel), S0, b, w for Gated DeltaNet-2.
Decode steps draw each step's q, k, v, x_alpha, x_beta from a generator
seeded with seed * 1_000_003 + step, so the whole decode sequence never has
to be held at once.

Tensors are returned on the CPU; callers move them where they need them.
"""
from dataclasses import dataclass
from typing import Optional

import torch
import torch.nn.functional as F

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "fwd" | "step" | "fwd_bwd" | "gdr2_fwd"
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str           # storage dtype of q, k, v, o ("f32" | "bf16")
    s0_std: float        # 0.0 means S0 = 0
    seed: int
    steps: int = 0       # decode steps (kind == "step")


# The five synthetic workloads the method is exercised on.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "fwd", 1, 128, 2, 64, 64, "f32", 0.0, 0),
    "layer_fwd": Workload("layer_fwd", "fwd", 4, 4096, 16, 128, 128, "bf16", 0.02, 1),
    "decode": Workload("decode", "step", 256, 1, 16, 128, 128, "bf16", 0.02, 2, steps=1024),
    "long_fwd_bwd": Workload("long_fwd_bwd", "fwd_bwd", 1, 65536, 16, 128, 128, "bf16", 0.0, 3),
    "gdn2_fwd": Workload("gdn2_fwd", "gdr2_fwd", 4, 4096, 16, 128, 128, "bf16", 0.02, 4),
}


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def gdr_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
               seed: int = 0, s0_std: float = 0.0, with_dO: bool = False) -> dict:
    """Inputs of the scalar-gate rule: q, k [B,T,H,dk], v [B,T,H,dv] in
    `dtype`; log_alpha, beta [B,T,H] fp32; S0 [B,H,dv,dk] fp32 or None;
    dO [B,T,H,dv] in `dtype` when with_dO."""
    g = torch.Generator().manual_seed(seed)
    dt = DTYPES[dtype]
    q = _l2n(torch.randn(B, T, H, dk, generator=g)).to(dt)
    k = _l2n(torch.randn(B, T, H, dk, generator=g)).to(dt)
    v = torch.randn(B, T, H, dv, generator=g).to(dt)
    log_alpha = -F.softplus(torch.randn(B, T, H, generator=g) - 2.0)
    beta = torch.sigmoid(torch.randn(B, T, H, generator=g))
    S0 = None
    if s0_std > 0.0:
        S0 = torch.randn(B, H, dv, dk, generator=g) * s0_std
    out = dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S0=S0)
    if with_dO:
        out["dO"] = torch.randn(B, T, H, dv, generator=g).to(dt)
    return out


def gdr2_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype: str = "bf16",
                seed: int = 0, s0_std: float = 0.0, b_max: float = 1.0) -> dict:
    """Inputs of Gated DeltaNet-2: q, k, v as above; log_alpha, b
    [B,T,H,dk] fp32; w [B,T,H,dv] fp32; S0 or None.  b = b_max * sigmoid(x):
    b_max = 2 gives the negative-eigenvalue range b in (0, 2)."""
    g = torch.Generator().manual_seed(seed)
    dt = DTYPES[dtype]
    q = _l2n(torch.randn(B, T, H, dk, generator=g)).to(dt)
    k = _l2n(torch.randn(B, T, H, dk, generator=g)).to(dt)
    v = torch.randn(B, T, H, dv, generator=g).to(dt)
    log_alpha = -F.softplus(torch.randn(B, T, H, dk, generator=g) - 2.0)
    S0 = None
    if s0_std > 0.0:
        S0 = torch.randn(B, H, dv, dk, generator=g) * s0_std
    b = b_max * torch.sigmoid(torch.randn(B, T, H, dk, generator=g))
    w = torch.sigmoid(torch.randn(B, T, H, dv, generator=g))
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, S0=S0)


def block_prologue_inputs(B: int, T: int, H: int, dk: int, dv: int, K: int, dtype: str = "bf16",
                          seed: int = 0, bias: bool = True, state: bool = True) -> dict:
    """Inputs of the block prologue (see the module docstring)."""
    g = torch.Generator().manual_seed(seed)
    dt = DTYPES[dtype]
    bound = 1.0 / K ** 0.5
    out = {}
    for n, d in (("xq", dk), ("xk", dk), ("xv", dv)):
        out[n] = torch.randn(B, T, H, d, generator=g).to(dt)
    for n, d in (("wq", dk), ("wk", dk), ("wv", dv)):
        out[n] = (torch.rand(H * d, K, generator=g) * 2 - 1) * bound
    for n, d in (("bq", dk), ("bk", dk), ("bv", dv)):
        out[n] = (torch.rand(H * d, generator=g) * 2 - 1) * bound if bias else None
    out["conv_state"] = (torch.randn(B, K - 1, H * (2 * dk + dv), generator=g).to(dt)
                         if state and K > 1 else None)
    return out


def block_prologue_bwd_inputs(B: int, T: int, H: int, dk: int, dv: int, K: int, dtype: str = "bf16",
                              seed: int = 0, bias: bool = True, state: bool = True,
                              dstate: bool = False) -> dict:
    """Prologue inputs plus incoming gradients dyq, dyk [B,T,H,dk], dyv
    [B,T,H,dv] ~ N(0, 1) in dtype and, with dstate, a gradient of the returned
    conv state dconv_state_out [B, K-1, H*(2dk+dv)] ~ N(0, 1)."""
    x = block_prologue_inputs(B, T, H, dk, dv, K, dtype, seed, bias, state)
    g = torch.Generator().manual_seed(seed * 7919 + 2)
    dt = DTYPES[dtype]
    for n, d in (("dyq", dk), ("dyk", dk), ("dyv", dv)):
        x[n] = torch.randn(B, T, H, d, generator=g).to(dt)
    x["dconv_state_out"] = (torch.randn(B, K - 1, H * (2 * dk + dv), generator=g).to(dt)
                            if dstate and K > 1 else None)
    return x


def block_epilogue_inputs(B: int, T: int, H: int, dv: int, dtype: str = "bf16", seed: int = 0,
                          gate: bool = True) -> dict:
    """Inputs of the block epilogue (see the module docstring)."""
    g = torch.Generator().manual_seed(seed)
    dt = DTYPES[dtype]
    o = (0.1 * torch.randn(B, T, H, dv, generator=g)).to(dt)
    gg = torch.randn(B, T, H, dv, generator=g).to(dt)
    weight = 1.0 + 0.1 * torch.randn(dv, generator=g)
    return {"o": o, "g": gg if gate else None, "weight": weight}


def block_epilogue_bwd_inputs(B: int, T: int, H: int, dv: int, dtype: str = "bf16", seed: int = 0,
                              gate: bool = True) -> dict:
    """Epilogue inputs plus an incoming gradient dy ~ N(0, 1) [B,T,H,dv] in dtype."""
    x = block_epilogue_inputs(B, T, H, dv, dtype, seed, gate)
    g = torch.Generator().manual_seed(seed * 7919 + 1)
    x["dy"] = torch.randn(B, T, H, dv, generator=g).to(DTYPES[dtype])
    return x


def decode_state(B: int, H: int, dk: int, dv: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """Initial decode state S [B,H,dv,dk] fp32 ~ N(0, std^2)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, H, dv, dk, generator=g) * std


def decode_step_inputs(B: int, H: int, dk: int, dv: int, dtype: str, seed: int,
                       step: int) -> dict:
    """One decode token for every (b,h): q, k [B,H,dk], v [B,H,dv] in dtype;
    log_alpha, beta [B,H] fp32."""
    g = torch.Generator().manual_seed(seed * 1_000_003 + step)
    dt = DTYPES[dtype]
    q = _l2n(torch.randn(B, H, dk, generator=g)).to(dt)
    k = _l2n(torch.randn(B, H, dk, generator=g)).to(dt)
    v = torch.randn(B, H, dv, generator=g).to(dt)
    log_alpha = -F.softplus(torch.randn(B, H, generator=g) - 2.0)
    beta = torch.sigmoid(torch.randn(B, H, generator=g))
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta)


def workload_inputs(name: str, T: Optional[int] = None) -> dict:
    """Inputs of a named workload (T overrides the sequence length, keeping
    the seed; the draws then differ from the full-length tensors)."""
    w = WORKLOADS[name]
    TT = w.T if T is None else T
    if w.kind == "gdr2_fwd":
        return gdr2_inputs(w.B, TT, w.H, w.dk, w.dv, w.dtype, w.seed, w.s0_std)
    return gdr_inputs(w.B, TT, w.H, w.dk, w.dv, w.dtype, w.seed, w.s0_std,
                      with_dO=(w.kind == "fwd_bwd"))
