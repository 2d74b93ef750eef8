"""Chunk-by-chunk streaming session over rehyat_chunk_forward_carry ("ReHyAt overview" page, §2.3:
the chunk-wise recurrent form, where only the linear state and the overlap frames are carried).

A session owns every device buffer it needs, allocated once when it is built: the state S
[B,H,F,D] and Z [B,H,F] (fp32), the carry (the last To frames of K and V seen, [B,H,To*L,D]) and
the workspace.  Each step is one library call on the incoming chunk: the library assembles the
softmax window from the carry and the chunk, attends, folds the frames the next window no longer
holds into S and Z, and updates the carry, so memory stays constant however long the video is.

Tc and To are the largest chunk and overlap the session accepts.  A step may pass a shorter
chunk and its own overlap (`To`) and the next step's (`To_next`): a variable schedule of the
"ReHyAt overview" page §5.2 (a longer first chunk, more overlap where motion is strong).

The session's state is its checkpoint: S, Z, the carry and the number of frames seen.
state_dict() copies it to host memory; load_state_dict() puts it back into a fresh session, and
the steps that follow produce the same bits as an uninterrupted run (same kernels, same order).
"""
from __future__ import annotations

import torch

from . import binding as rb


class ChunkStream:
    def __init__(self, Wq, bq, Wk, bk, *, B: int, P: int, frame_tokens: int, Tc: int, To: int,
                 phi: int = rb.PHI_POLY, dtype: torch.dtype = torch.bfloat16,
                 device: torch.device | None = None):
        dev = device or Wq.device
        H, G, Fg, Dg = Wq.shape
        D, F = Dg * G, Fg * G
        self.Wq, self.bq, self.Wk, self.bk = Wq, bq, Wk, bk
        self.B, self.H, self.D, self.F, self.P, self.phi = B, H, D, F, P, phi
        self.L, self.Tc, self.To = frame_tokens, Tc, To
        self.dtype, self.device = dtype, dev
        self.frames_seen = 0
        self.S = torch.zeros(B, H, F, D, dtype=torch.float32, device=dev)
        self.Z = torch.zeros(B, H, F, dtype=torch.float32, device=dev)
        self.k_carry = torch.zeros(B, H, To * frame_tokens, D, dtype=dtype, device=dev)
        self.v_carry = torch.zeros_like(self.k_carry)
        d = rb.Dims(B, H, D, F, G, P, phi)
        code = rb.REHYAT_BF16 if dtype == torch.bfloat16 else rb.REHYAT_F32
        self.workspace = torch.empty(rb.chunk_carry_workspace_size(d, code, frame_tokens, Tc, To,
                                                                   To),
                                     dtype=torch.uint8, device=dev)

    def reset(self) -> None:
        """Start a new sequence (the buffers are kept)."""
        self.S.zero_()
        self.Z.zero_()
        self.frames_seen = 0

    def step(self, q, k, v, out: torch.Tensor | None = None, To: int | None = None,
             To_next: int | None = None) -> torch.Tensor:
        """Attend the next chunk (q, k, v: [B,H,chunk_frames*L,D], 1 <= chunk_frames <= Tc);
        returns its output [B,H,chunk_frames*L,D].  To / To_next: this chunk's and the next
        chunk's overlap (default: the session's To)."""
        L, cap = self.L, self.To
        To = cap if To is None else To
        n = q.shape[2]
        if n % L or not 1 <= n // L <= self.Tc or k.shape != q.shape or v.shape != q.shape:
            raise ValueError(f"chunk of {n} rows is not 1..{self.Tc} frames of {L} tokens")
        if not 0 <= To <= cap or (To_next is not None and not 0 <= To_next <= cap):
            raise ValueError(f"overlaps must lie in [0, {cap}]")
        out = rb.chunk_forward_carry(q, k, v, self.Wq, self.bq, self.Wk, self.bk, self.S, self.Z,
                                     self.k_carry, self.v_carry, P=self.P, phi=self.phi,
                                     frame_tokens=L, frames_before=self.frames_seen, To=To,
                                     To_next=To_next, out=out, workspace=self.workspace)
        self.frames_seen += n // L
        return out

    def state_dict(self) -> dict:
        """The session's state, copied to host memory."""
        return {"S": self.S.cpu(), "Z": self.Z.cpu(), "k_carry": self.k_carry.cpu(),
                "v_carry": self.v_carry.cpu(), "frames_seen": self.frames_seen,
                "shape": (self.B, self.H, self.D, self.F, self.P, self.L, self.Tc, self.To,
                          self.phi)}

    def load_state_dict(self, st: dict) -> None:
        if tuple(st["shape"]) != (self.B, self.H, self.D, self.F, self.P, self.L, self.Tc,
                                  self.To, self.phi):
            raise ValueError(f"state of shape {st['shape']} does not fit this session")
        self.S.copy_(st["S"])
        self.Z.copy_(st["Z"])
        self.k_carry.copy_(st["k_carry"])
        self.v_carry.copy_(st["v_carry"])
        self.frames_seen = int(st["frames_seen"])
