"""Chunk-by-chunk streaming session over rehyat_chunk_forward ("ReHyAt overview" page, §2.3:
the chunk-wise recurrent form, where only the linear state and the overlap frames are carried).

A session owns every device buffer it needs, allocated once when it is built: the state S
[B,H,F,D] and Z [B,H,F] (fp32), the last To frames of K and V (two buffers used in turn), the
window buffers that rehyat_chunk_forward reads ([B,H,(overlap + chunk) frames,D], contiguous),
and the workspace.  Each step copies the incoming chunk into the window behind the saved
overlap frames, runs the C call, and keeps the last To frames seen for the next step, so memory
stays constant however long the video is.

Tc and To are the largest chunk and overlap the session accepts.  A step may pass a shorter
chunk and its own overlap (`To`) and the next step's (`To_next`): a variable schedule of the
"ReHyAt overview" page §5.2 (a longer first chunk, more overlap where motion is strong).

The session's state is its checkpoint: S, Z, the overlap frames and the number of frames seen.
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
        self.k_tail = torch.zeros(B, H, To * frame_tokens, D, dtype=dtype, device=dev)
        self.v_tail = torch.zeros_like(self.k_tail)
        self._k_spare = torch.zeros_like(self.k_tail)
        self._v_spare = torch.zeros_like(self.k_tail)
        cap = B * H * (To + Tc) * frame_tokens * D
        self._k_flat = torch.empty(cap, dtype=dtype, device=dev)
        self._v_flat = torch.empty(cap, dtype=dtype, device=dev)
        d = rb.Dims(B, H, D, F, G, P, phi)
        code = rb._dtype_code(self._k_flat)
        self.workspace = torch.empty(rb.chunk_workspace_size(d, code, frame_tokens, Tc, To),
                                     dtype=torch.uint8, device=dev)

    def _window(self, flat: torch.Tensor, rows: int) -> torch.Tensor:
        return flat[:self.B * self.H * rows * self.D].view(self.B, self.H, rows, self.D)

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
        cf = n // L
        ov = min(To, self.frames_seen)
        rows = (ov + cf) * L
        kw, vw = self._window(self._k_flat, rows), self._window(self._v_flat, rows)
        if ov:
            kw[:, :, :ov * L].copy_(self.k_tail[:, :, (cap - ov) * L:])
            vw[:, :, :ov * L].copy_(self.v_tail[:, :, (cap - ov) * L:])
        kw[:, :, ov * L:].copy_(k)
        vw[:, :, ov * L:].copy_(v)
        out = rb.chunk_forward(q, kw, vw, self.Wq, self.bq, self.Wk, self.bk, self.S, self.Z,
                               P=self.P, phi=self.phi, frame_tokens=L,
                               frames_before=self.frames_seen, To=To, To_next=To_next,
                               out=out, workspace=self.workspace)
        # the last `cap` frames seen, at the end of the tail (fewer at the start), built in the
        # spare buffer from the old tail shifted by the chunk, then the buffers swap
        if cap:
            for tail, spare, x in ((self.k_tail, self._k_spare, k), (self.v_tail, self._v_spare, v)):
                if cf >= cap:
                    spare.copy_(x[:, :, (cf - cap) * L:])
                else:
                    spare[:, :, :(cap - cf) * L].copy_(tail[:, :, cf * L:])
                    spare[:, :, (cap - cf) * L:].copy_(x)
            self.k_tail, self._k_spare = self._k_spare, self.k_tail
            self.v_tail, self._v_spare = self._v_spare, self.v_tail
        self.frames_seen += cf
        return out

    def state_dict(self) -> dict:
        """The session's state, copied to host memory."""
        return {"S": self.S.cpu(), "Z": self.Z.cpu(), "k_tail": self.k_tail.cpu(),
                "v_tail": self.v_tail.cpu(), "frames_seen": self.frames_seen,
                "shape": (self.B, self.H, self.D, self.F, self.P, self.L, self.Tc, self.To,
                          self.phi)}

    def load_state_dict(self, st: dict) -> None:
        if tuple(st["shape"]) != (self.B, self.H, self.D, self.F, self.P, self.L, self.Tc,
                                  self.To, self.phi):
            raise ValueError(f"state of shape {st['shape']} does not fit this session")
        self.S.copy_(st["S"])
        self.Z.copy_(st["Z"])
        self.k_tail.copy_(st["k_tail"])
        self.v_tail.copy_(st["v_tail"])
        self.frames_seen = int(st["frames_seen"])
