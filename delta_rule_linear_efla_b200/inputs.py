"""Seeded synthetic inputs for the EFLA forward workloads.

This module holds only input distributions: it draws q, k, v, beta and the
initial state on the host with a seeded torch CPU generator and rounds them to
the workload's dtype.  It contains none of the method's arithmetic, so both
the CUDA path and the CPU oracle can be fed from it.

Workloads (shapes, dtypes and value distributions):

  id  name               B   H     L  dk=dv chunk dtype  q                   k                       beta          S0
  1   tiny-fp32          1   1    64   16   16   fp32   N(0,1/dk)*LU[.1,3]  N(0,1/dk)*LU[.1,3]      sig(N(0,1))   0
  2   small-bf16         2   4  1024   64   64   bf16   N(0,1/dk)*LU[.5,2]  N(0,1/dk)*LU[.5,2]      sig(N(0,1))   N(0,0.01)
  3   lm340m-bf16        8   8  2048  128   64   bf16   N(0,1/dk)           ||k||^2 ~ LU[0.25,4]    sig(N(0,1))   0
  4   lm1p3b-bf16        4  16  4096  128   64   bf16   N(0,1/dk)*LU[.5,2]  ||k||^2 ~ LU[0.25,4]    sig(N(0,1))   0
  5   long-stiff-bf16    1  16 65536  128   64   bf16   N(0,1/dk)           ||k||^2 ~ LU[1e-4,100]  sig(N(0,4))   0

v ~ N(0,1) everywhere; in workload 5 a seeded 5% of the (b, t) positions have
v scaled by 10 for every head (high-energy inputs).  N(m, s) names the
variance s.  LU[a,b] is log-uniform: exp(U(ln a, ln b)), drawn per (b, h, t)
and independently for q and k.  "||k||^2 ~ LU" draws a direction uniformly on
the sphere (a normalised Gaussian) and a squared norm from LU.

Workload 4 also carries a decode batch: B=64 sequences, H=16, one token each,
after a 256-token prefix drawn with workload-4 distributions (seed 2004).  The
prefix's final state is the carried fp32 state the decode step starts from.

The default seed of workload i is 1000 + i.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    id: int
    name: str
    B: int
    H: int
    L: int
    dk: int
    dv: int
    chunk: int
    dtype: str  # "fp32" or "bf16"
    q: tuple  # ("gauss",) | ("gauss_lu", a, b)
    k: tuple  # ("gauss_lu", a, b) | ("norm2_lu", a, b)
    beta_std: float
    s0_std: float
    v_hi: tuple | None = None  # (fraction, scale)
    decode: dict | None = field(default=None, compare=False)

    @property
    def token_heads(self) -> int:
        return self.B * self.H * self.L

    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16


WORKLOADS = {
    1: Workload(1, "tiny-fp32", 1, 1, 64, 16, 16, 16, "fp32",
                ("gauss_lu", 0.1, 3.0), ("gauss_lu", 0.1, 3.0), 1.0, 0.0),
    2: Workload(2, "small-bf16", 2, 4, 1024, 64, 64, 64, "bf16",
                ("gauss_lu", 0.5, 2.0), ("gauss_lu", 0.5, 2.0), 1.0, 0.1),
    3: Workload(3, "lm340m-bf16", 8, 8, 2048, 128, 128, 64, "bf16",
                ("gauss",), ("norm2_lu", 0.25, 4.0), 1.0, 0.0),
    4: Workload(4, "lm1p3b-bf16", 4, 16, 4096, 128, 128, 64, "bf16",
                ("gauss_lu", 0.5, 2.0), ("norm2_lu", 0.25, 4.0), 1.0, 0.0,
                decode=dict(B=64, H=16, prefix=256, seed=2004)),
    5: Workload(5, "long-stiff-bf16", 1, 16, 65536, 128, 128, 64, "bf16",
                ("gauss",), ("norm2_lu", 1e-4, 100.0), 2.0, 0.0, v_hi=(0.05, 10.0)),
}


def workload(wid: int, **overrides) -> Workload:
    """The named workload, optionally with some fields replaced (e.g. L=200)."""
    return replace(WORKLOADS[wid], **overrides)


def _log_uniform(g: torch.Generator, shape, a: float, b: float) -> torch.Tensor:
    u = torch.rand(shape, generator=g, dtype=torch.float32)
    return torch.exp(math.log(a) + (math.log(b) - math.log(a)) * u)


def _vectors(g: torch.Generator, spec: tuple, B: int, H: int, L: int, d: int) -> torch.Tensor:
    kind = spec[0]
    x = torch.randn((B, H, L, d), generator=g, dtype=torch.float32)
    if kind == "gauss":
        x.mul_(1.0 / math.sqrt(d))
    elif kind == "gauss_lu":
        x.mul_(1.0 / math.sqrt(d))
        x.mul_(_log_uniform(g, (B, H, L, 1), spec[1], spec[2]))
    elif kind == "norm2_lu":
        x.div_(x.norm(dim=-1, keepdim=True).clamp_min(1e-30))
        x.mul_(_log_uniform(g, (B, H, L, 1), spec[1], spec[2]).sqrt_())
    else:
        raise ValueError(kind)
    return x


def make_inputs(w: Workload | int, seed: int | None = None) -> dict:
    """Host tensors {q, k, v, beta, S0} for a workload, rounded to its dtype.

    q, k: [B,H,L,dk]; v: [B,H,L,dv]; beta: [B,H,L] (all in the workload dtype);
    S0: [B,H,dk,dv] fp32 or None when the workload starts from zeros.
    """
    if isinstance(w, int):
        w = WORKLOADS[w]
    g = torch.Generator().manual_seed(1000 + w.id if seed is None else seed)
    dt = w.torch_dtype()
    q = _vectors(g, w.q, w.B, w.H, w.L, w.dk).to(dt)
    k = _vectors(g, w.k, w.B, w.H, w.L, w.dk).to(dt)
    v = torch.randn((w.B, w.H, w.L, w.dv), generator=g, dtype=torch.float32)
    if w.v_hi is not None:
        frac, scale = w.v_hi
        hi = torch.rand((w.B, 1, w.L, 1), generator=g) < frac
        v = torch.where(hi, v * scale, v)
    v = v.to(dt)
    beta = torch.sigmoid(w.beta_std * torch.randn((w.B, w.H, w.L), generator=g,
                                                  dtype=torch.float32)).to(dt)
    S0 = None
    if w.s0_std > 0:
        S0 = w.s0_std * torch.randn((w.B, w.H, w.dk, w.dv), generator=g, dtype=torch.float32)
    return dict(q=q, k=k, v=v, beta=beta, S0=S0, chunk=w.chunk, workload=w)


def make_gate(shape, dtype, seed: int) -> torch.Tensor:
    """Per-token decays for the gated form, sigmoid(N(2, 1)) (mean about 0.86, a few tokens near
    0.5), drawn with their own seeded generator and rounded to `dtype`."""
    g = torch.Generator().manual_seed(seed)
    return torch.sigmoid(2.0 + torch.randn(shape, generator=g, dtype=torch.float32)).to(dtype)


def make_decode_inputs(w: Workload | int = 4, seed: int | None = None) -> dict:
    """Decode batch of a workload that carries one (workload 4).

    Returns {prefix: make_inputs(...) of the 256-token prefix, q, k, v, beta}
    where q, k: [B,H,dk], v: [B,H,dv], beta: [B,H] for the one new token.  The
    carried state is the prefix's final state, computed by the caller.
    """
    if isinstance(w, int):
        w = WORKLOADS[w]
    dec = w.decode
    if dec is None:
        raise ValueError("workload %d has no decode batch" % w.id)
    s = dec["seed"] if seed is None else seed
    pw = replace(w, B=dec["B"], H=dec["H"], L=dec["prefix"] + 1, decode=None)
    full = make_inputs(pw, seed=s)
    P = dec["prefix"]
    prefix = dict(full)
    for name in ("q", "k", "v"):
        prefix[name] = full[name][:, :, :P].contiguous()
    prefix["beta"] = full["beta"][:, :, :P].contiguous()
    prefix["workload"] = replace(pw, L=P)
    return dict(prefix=prefix,
                q=full["q"][:, :, P].contiguous(), k=full["k"][:, :, P].contiguous(),
                v=full["v"][:, :, P].contiguous(), beta=full["beta"][:, :, P].contiguous(),
                workload=pw)
