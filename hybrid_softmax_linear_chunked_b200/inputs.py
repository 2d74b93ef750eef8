"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

Holds random-number generation only, none of the method's arithmetic.  Draw order on one CPU
torch.Generator: q, k, v, then W_q, W_k (fp32 normal); biases are constant fills.
"""
from __future__ import annotations

import dataclasses

import torch

from .configs import Workload, weight_std


@dataclasses.dataclass
class Inputs:
    q: torch.Tensor    # [B, H, N, D] (dtype of the workload), CPU
    k: torch.Tensor
    v: torch.Tensor
    Wq: torch.Tensor   # [H, G, F/G, D/G] fp32
    bq: torch.Tensor   # [H, F] fp32
    Wk: torch.Tensor
    bk: torch.Tensor


def make_inputs(w: Workload, seed: int | None = None, heads: int | None = None,
                batch: int | None = None, frames: int | None = None) -> Inputs:
    """Generate the workload's inputs on the CPU.  `heads`/`batch`/`frames` cut the problem down
    (the values drawn for the kept part depend on the cut, so only compare cuts made the same
    way)."""
    B = w.B if batch is None else batch
    H = w.H if heads is None else heads
    T = w.T if frames is None else frames
    N = T * w.frame_tokens
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q = torch.randn(B, H, N, w.D, generator=g).to(dt)
    k = torch.randn(B, H, N, w.D, generator=g).to(dt)
    v = torch.randn(B, H, N, w.D, generator=g).to(dt)
    if w.k_scale != 1.0:
        k = (k.float() * w.k_scale).to(dt)
    std = weight_std(w)
    Wq = torch.randn(H, w.G, w.F // w.G, w.D // w.G, generator=g) * std
    Wk = torch.randn(H, w.G, w.F // w.G, w.D // w.G, generator=g) * std
    bq = torch.full((H, w.F), float(w.bias))
    bk = torch.full((H, w.F), float(w.bias))
    return Inputs(q, k, v, Wq, bq, Wk, bk)
