"""Seeded synthetic inputs for the gated delta-rule operator.

This module draws the random tensors that both the CUDA path and the CPU oracle
consume.  It holds none of the operator's arithmetic: it only samples, shapes,
normalises and rounds inputs, following the workload recipe of the five
workloads below.

Recipe (one CPU ``torch.Generator`` seeded with ``seed``; draws in this order):
  q, k ~ N(0, 1)  [B, T, H, Dk], then L2-normalised over Dk in fp32
  v    ~ N(0, 1)  [B, T, H, Dv]
  beta = sigmoid(N(0, 1))          [B, T, H]
  g    = -softplus(N(0, 1)) * c    [B, T, H] (scalar gate) or [B, T, H, Dk]
         (per-dimension gate); g = log a, so a = exp(g) in (0, 1]
  S0   = s0_std * N(0, 1)          [B, H, Dk, Dv] fp32 (or absent)
Every token tensor is then rounded to the workload dtype (bf16 or fp32);
states stay fp32.  The decode workload draws its 128 tokens per sequence the
same way with B = number of sequences and T = number of decode steps.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.nn.functional as F

GATE_NONE, GATE_SCALAR, GATE_PER_DIM = 0, 1, 2
GATE_NAMES = {"none": GATE_NONE, "scalar": GATE_SCALAR, "per_dim": GATE_PER_DIM}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "chunk" or "decode"
    B: int             # batch (decode: number of sequences)
    T: int             # tokens (decode: number of consecutive decode steps)
    H: int
    Dk: int
    Dv: int
    chunk: int
    dtype: str         # "bf16" or "f32" (token dtype; states are always fp32)
    gate: str          # "none", "scalar" or "per_dim"
    gate_scale: float  # c in g = -softplus(x) * c
    s0_std: float | None
    seed: int = 0

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def gate_kind(self) -> int:
        return GATE_NAMES[self.gate]


WORKLOADS = {
    0: Workload("tiny delta-rule fwd fp32 B1 H2 T256 d64", "chunk",
                1, 256, 2, 64, 64, 64, "f32", "scalar", 0.1, None),
    1: Workload("GDN scalar-gated chunk fwd bf16 B4 H16 T2048 d128", "chunk",
                4, 2048, 16, 128, 128, 64, "bf16", "scalar", 0.1, None),
    2: Workload("KDA per-dim-gated chunk fwd bf16 B4 H16 T4096 d128", "chunk",
                4, 4096, 16, 128, 128, 64, "bf16", "per_dim", 0.05, 0.02),
    3: Workload("long-sequence scalar-gated chunk fwd bf16 B1 H32 T65536 d128", "chunk",
                1, 65536, 32, 128, 128, 64, "bf16", "scalar", 0.1, None),
    4: Workload("recurrent decode N256 H32 d128 x128 steps", "decode",
                256, 128, 32, 128, 128, 64, "bf16", "scalar", 0.1, 0.02),
}


def make_inputs(B: int, T: int, H: int, Dk: int, Dv: int, *, dtype=torch.bfloat16,
                gate: str = "scalar", gate_scale: float = 0.1,
                s0_std: float | None = None, seed: int = 0, device="cpu") -> dict:
    """Draw one seeded input set.  Returns a dict of tensors on `device`:
    q, k, v, beta, g (None for gate "none"), S0 (None when s0_std is None),
    plus ``gate_kind`` (int).  The recipe is the same on every device; the
    random stream is the device's own, so a CUDA draw gives other values than
    the CPU draw of the same seed (the parity tests use the CPU draw)."""
    gen = torch.Generator(device=device).manual_seed(seed)
    kw = dict(generator=gen, device=device)
    q = torch.randn(B, T, H, Dk, **kw)
    k = torch.randn(B, T, H, Dk, **kw)
    v = torch.randn(B, T, H, Dv, **kw)
    beta_logit = torch.randn(B, T, H, **kw)
    g = None
    if gate == "scalar":
        g = -F.softplus(torch.randn(B, T, H, **kw)) * gate_scale
    elif gate == "per_dim":
        g = -F.softplus(torch.randn(B, T, H, Dk, **kw)) * gate_scale
    elif gate != "none":
        raise ValueError(f"unknown gate {gate!r}")
    S0 = None
    if s0_std is not None:
        S0 = (torch.randn(B, H, Dk, Dv, **kw) * s0_std).contiguous()
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    beta = torch.sigmoid(beta_logit)
    out = {
        "q": q.to(dtype).contiguous(),
        "k": k.to(dtype).contiguous(),
        "v": v.to(dtype).contiguous(),
        "beta": beta.to(dtype).contiguous(),
        "g": None if g is None else g.to(dtype).contiguous(),
        "S0": S0,
        "gate_kind": GATE_NAMES[gate],
    }
    return out


def workload_inputs(w: Workload, *, T: int | None = None, B: int | None = None,
                    H: int | None = None, seed: int | None = None, device="cpu") -> dict:
    """Inputs of a named workload; T/B/H (and the seed) may be overridden for
    a reduced case or one rank's share of the heads."""
    return make_inputs(w.B if B is None else B, w.T if T is None else T,
                       w.H if H is None else H, w.Dk, w.Dv, dtype=w.torch_dtype, gate=w.gate,
                       gate_scale=w.gate_scale, s0_std=w.s0_std,
                       seed=w.seed if seed is None else seed, device=device)


def to_f64_numpy(inputs: dict) -> dict:
    """The same tensors widened to float64 numpy arrays (exact: every bf16/fp32
    value is representable in fp64)."""
    import numpy as np
    out = {}
    for key, val in inputs.items():
        if isinstance(val, torch.Tensor):
            out[key] = val.to(torch.float64).numpy()
        else:
            out[key] = val
    return out
