"""Workload descriptions of the hybrid attention forward (shapes, schedule and input recipe).

Pure data: nothing here computes any part of the method.
"""
from __future__ import annotations

import dataclasses
import math


@dataclasses.dataclass(frozen=True)
class Workload:
    """One hybrid-attention problem.

    B, H           : batch and heads; every (b, h) is an independent problem.
    D              : head dimension of q, k, v.
    T, frame_h, frame_w : latent frames and the spatial token grid of one frame
                     (frame_tokens = frame_h * frame_w tokens per frame, frame-major order).
    Tc, To, P      : chunk length in frames, overlap frames before the chunk, polynomial parts.
    F, G           : feature count of phi and the group count of its grouped 1x1 linear.
    dtype          : "f32" or "bf16" for q, k, v and the output.
    k_scale        : k is multiplied by this after rounding to dtype (exact for powers of two).
    bias           : constant filled into the feature-map biases (0 in the standard workloads).
    seed           : generator seed.
    mode           : "full" (one call over the sequence) or "stream" (chunk-by-chunk calls).
    phi            : feature map after the grouped linear: "poly" (softplus parts raised to
                     powers 1..P) or "elu1" (elu + 1).
    """
    name: str
    B: int
    H: int
    D: int
    T: int
    frame_h: int
    frame_w: int
    Tc: int
    To: int
    P: int
    F: int
    G: int
    dtype: str
    k_scale: float = 1.0
    bias: float = 0.0
    seed: int = 0
    mode: str = "full"
    phi: str = "poly"

    @property
    def phi_code(self) -> int:
        """The rehyat_phi value of `phi` (0 polynomial, 1 elu + 1)."""
        return {"poly": 0, "elu1": 1}[self.phi]

    @property
    def frame_tokens(self) -> int:
        return self.frame_h * self.frame_w

    @property
    def N(self) -> int:
        return self.T * self.frame_tokens

    @property
    def n_chunks(self) -> int:
        return -(-self.T // self.Tc)

    def chunk_bounds(self):
        """(w_c, s_c, e_c) frame bounds of each chunk: softmax window [w_c, e_c), queries
        [s_c, e_c)."""
        out = []
        for c in range(self.n_chunks):
            s = c * self.Tc
            e = min(s + self.Tc, self.T)
            out.append((max(0, s - self.To), s, e))
        return out

    def flops(self, streaming: bool | None = None) -> float:
        """Algorithmic FLOPs of one forward over all (b, h): softmax QK^T and PV over each
        chunk's window, the phi_q . S / phi_q . Z readout of chunks that have a linear region,
        the state fold, and the feature maps (2 D F / G per token per map) of the queries that
        read a state and the keys that are folded.  Exponentials and
        softplus count zero.  The full-sequence call folds only what a later chunk reads; the
        streaming calls fold after every chunk."""
        streaming = (self.mode == "stream") if streaming is None else streaming
        L, D, F = self.frame_tokens, self.D, self.F
        bounds = self.chunk_bounds()
        tot = 0.0
        folded = 0
        phi_q_tokens = 0
        for c, (w, s, e) in enumerate(bounds):
            nq, nw = (e - s) * L, (e - w) * L
            tot += 4.0 * nq * nw * D
            if w > 0:
                tot += nq * (2.0 * F * D + 2.0 * F)
                phi_q_tokens += nq
            if c + 1 < len(bounds):
                folded += (bounds[c + 1][0] - w) * L
            elif streaming:
                folded += (max(0, e - self.To) - w) * L
        tot += folded * (2.0 * F * D + F)
        tot += (phi_q_tokens + folded) * 2.0 * D * F / self.G
        return tot * self.B * self.H

    def attn_tensor_flops(self) -> float:
        """Tensor-core FLOPs of the fused attention kernel over all (b, h): Q K^T and P V over
        each chunk's window and the phi_q . S readout (2 F D per query of a chunk that has a
        linear region).  The CUDA-core work in the same kernel (phi_q, phi_q . Z, softmax) is
        not counted."""
        L, D, F = self.frame_tokens, self.D, self.F
        tot = 0.0
        for (w, s, e) in self.chunk_bounds():
            nq, nw = (e - s) * L, (e - w) * L
            tot += 4.0 * nq * nw * D
            if w > 0:
                tot += 2.0 * nq * F * D
        return tot * self.B * self.H

    def backward_flops(self) -> float:
        """Algorithmic FLOPs of the backward over all (b, h): QK^T, dO V^T, dS K, dS^T Q and
        P^T dO over each chunk's window; dO S_c^T and (lam phi_q)^T dO for chunks with a linear
        region; V R~^T and phi_k R~ for the keys read linearly; and the grouped linear of each
        feature map three times (u, dx, dW: 2 D F / G per token each)."""
        L, D, F = self.frame_tokens, self.D, self.F
        bounds = self.chunk_bounds()
        tot = 0.0
        q_rows = 0
        for (w, s, e) in bounds:
            nq, nw = (e - s) * L, (e - w) * L
            tot += 10.0 * nq * nw * D
            if w > 0:
                tot += 4.0 * nq * D * F
                q_rows += nq
        k_rows = bounds[-1][0] * L
        tot += 4.0 * k_rows * D * F
        tot += 3 * 2.0 * (q_rows + k_rows) * D * F / self.G
        return tot * self.B * self.H

    def io_bytes(self) -> float:
        """Algorithmic HBM bytes: q, k, v read once and the output written once."""
        el = 4 if self.dtype == "f32" else 2
        return 4.0 * self.B * self.H * self.N * self.D * el


TINY_F32 = Workload("tiny fp32 (6 frames x 4x4 tokens)", B=1, H=1, D=32, T=6, frame_h=4,
                    frame_w=4, Tc=3, To=1, P=2, F=32, G=4, dtype="f32")
WAN_480P_5S = Workload("480x832 5 s (21 frames x 30x52 tokens, 12 heads)", B=1, H=12, D=128,
                       T=21, frame_h=30, frame_w=52, Tc=3, To=1, P=2, F=128, G=8, dtype="bf16")
WAN_480P_10S = Workload("480x832 10 s (41 frames x 30x52 tokens, 12 heads)", B=1, H=12, D=128,
                        T=41, frame_h=30, frame_w=52, Tc=3, To=1, P=2, F=128, G=8, dtype="bf16")
WAN_720P_5S = Workload("720x1280 5 s (21 frames x 45x80 tokens, 12 heads, k x2)", B=1, H=12,
                       D=128, T=21, frame_h=45, frame_w=80, Tc=3, To=1, P=2, F=128, G=8,
                       dtype="bf16", k_scale=2.0)
WAN_480P_20S_STREAM = Workload("480x832 20 s streaming (B=2, 81 frames x 30x52 tokens)", B=2,
                               H=12, D=128, T=81, frame_h=30, frame_w=52, Tc=3, To=1, P=2,
                               F=128, G=8, dtype="bf16", mode="stream")

ALL = [TINY_F32, WAN_480P_5S, WAN_480P_10S, WAN_720P_5S, WAN_480P_20S_STREAM]


def ablation(Tc: int, To: int, P: int) -> Workload:
    """The 21-frame 480x832 shape with another chunk length, overlap or part count."""
    return dataclasses.replace(WAN_480P_5S, name=f"480x832 5 s Tc={Tc} To={To} P={P}", Tc=Tc,
                               To=To, P=P)


def weight_std(w: Workload) -> float:
    """Feature-map weights are N(0, 1/(D/G)) (variance), i.e. std sqrt(G/D)."""
    return math.sqrt(w.G / w.D)
