"""Context parallelism: one sequence split into contiguous chunk ranges, one range per GPU.

The state chunk c reads is the sum of the folds of every earlier chunk ("ReHyAt overview" page
§2.3), so a sequence cut at chunk boundaries couples its pieces through two things only:
  * the To overlap frames of K and V that the first chunk of a range takes from the range before
    it (the halo), sent point to point from rank r-1 to rank r;
  * the sum of the folds of all earlier ranges: each rank computes the sum of its own folds, the
    sums are all-gathered, and each rank adds those of the ranks before it (in the scan kernel,
    in rank order).
Everything else (feature maps, folds, scans, attention) runs locally through the library's
two-phase segment calls.

Each rank holds its own frames [s0, s1) of q and of k, v; k and v sit in buffers with room for
the halo in front ([h0, s1) with h0 = max(0, s0 - To)), see `ContextParallel.kv_buffer`.  The
process group must be initialised by the caller (NCCL for GPUs); every rank takes the same
collective steps in the same order.  The compute calls come from `ops` (the library binding by
default), so the host logic can be exercised with stand-in compute.
"""
from __future__ import annotations

import torch

from . import binding as rb


def split_chunks(C: int, world: int) -> list[tuple[int, int]]:
    """Contiguous chunk ranges [c0, c1), one per rank, as even as possible (the first C % world
    ranks get one chunk more).  Needs C >= world."""
    if world < 1 or C < world:
        raise ValueError(f"{C} chunks cannot be split over {world} ranks")
    base, extra = divmod(C, world)
    out, c0 = [], 0
    for r in range(world):
        c1 = c0 + base + (1 if r < extra else 0)
        out.append((c0, c1))
        c0 = c1
    return out


def plan_ranks(T: int, Tc: int, To: int, world: int):
    """Chunk ranges and (s0, s1, h0) bounds of every rank.  Raises ValueError when a rank holds
    fewer frames than the overlap the next rank takes from it (its halo must come from one
    rank)."""
    C = (T + Tc - 1) // Tc
    ranges = split_chunks(C, world)
    bounds = [rb.segment_bounds(T, Tc, To, c0, c1) for c0, c1 in ranges]
    for r in range(world - 1):
        s0, s1, _ = bounds[r]
        n0, _, nh = bounds[r + 1]
        if s1 - s0 < n0 - nh:
            raise ValueError(f"rank {r} holds {s1 - s0} frames, fewer than the {n0 - nh} overlap "
                             "frames the next rank needs")
    return ranges, bounds


class ContextParallel:
    """The forward of one sequence of T frames over the ranks of `group` (or one process)."""

    def __init__(self, Wq, bq, Wk, bk, *, T: int, frame_tokens: int, Tc: int, To: int, P: int,
                 phi: int = rb.PHI_POLY, group=None, ops=None):
        import torch.distributed as dist
        self.dist = dist if dist.is_available() and dist.is_initialized() else None
        self.group = group
        self.rank = self.dist.get_rank(group) if self.dist else 0
        self.world = self.dist.get_world_size(group) if self.dist else 1
        self.ops = ops if ops is not None else rb
        self.Wq, self.bq, self.Wk, self.bk = Wq, bq, Wk, bk
        self.T, self.L, self.Tc, self.To, self.P, self.phi = T, frame_tokens, Tc, To, P, phi
        self.C = (T + Tc - 1) // Tc
        self.ranges, self.bounds = plan_ranks(T, Tc, To, self.world)
        self.c0, self.c1 = self.ranges[self.rank]
        self.s0, self.s1, self.h0 = self.bounds[self.rank]
        self._ws = None
        self._dims = None

    # ---- layout ----
    def halo_frames(self, r: int) -> int:
        s0, _, h0 = self.bounds[r]
        return s0 - h0

    def kv_buffer(self, like: torch.Tensor) -> torch.Tensor:
        """A [B,H,(s1-h0)*L,D] buffer for this rank's k or v; the own frames go to
        `own(buf)`, the halo is filled by `forward`."""
        B, H, _, D = like.shape
        return torch.empty(B, H, (self.s1 - self.h0) * self.L, D, dtype=like.dtype,
                           device=like.device)

    def own(self, buf: torch.Tensor) -> torch.Tensor:
        """The view of this rank's own frames [s0, s1) in a kv_buffer."""
        return buf[:, :, (self.s0 - self.h0) * self.L:]

    # ---- exchange ----
    def _exchange_halo(self, bufs: list[torch.Tensor]) -> None:
        """Rank r-1 sends the last halo frames of its own k, v to rank r (point to point)."""
        if self.dist is None or self.world == 1:
            return
        dist, L = self.dist, self.L
        ops, recv_bufs = [], []
        h_in = self.halo_frames(self.rank)
        if self.rank > 0 and h_in > 0:
            for b in bufs:
                t = torch.empty_like(b[:, :, :h_in * L]).contiguous()
                recv_bufs.append((b, t))
                ops.append(dist.P2POp(dist.irecv, t, self._peer(self.rank - 1), self.group))
        if self.rank + 1 < self.world:
            h_out = self.halo_frames(self.rank + 1)
            if h_out > 0:
                for b in bufs:
                    t = b[:, :, b.shape[2] - h_out * L:].contiguous()
                    ops.append(dist.P2POp(dist.isend, t, self._peer(self.rank + 1), self.group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
        for b, t in recv_bufs:
            b[:, :, :t.shape[2]].copy_(t)

    def _peer(self, r: int) -> int:
        """Global rank of group rank r."""
        if self.group is None:
            return r
        return self.dist.get_global_rank(self.group, r)

    def _all_gather(self, x: torch.Tensor) -> torch.Tensor:
        if self.dist is None or self.world == 1:
            return x.unsqueeze(0)
        parts = [torch.empty_like(x) for _ in range(self.world)]
        self.dist.all_gather(parts, x.contiguous(), group=self.group)
        return torch.stack(parts)

    # ---- forward ----
    def workspace(self, device) -> torch.Tensor:
        """The segment workspace (allocated once per device, reused by every forward)."""
        if self._ws is None or self._ws.device != torch.device(device):
            n = self.ops.segment_workspace_size(self._dims, self.T, self.L, self.Tc, self.To,
                                                self.c0, self.c1)
            self._ws = torch.empty(max(n, 16), dtype=torch.uint8, device=device)
        return self._ws

    def forward(self, q_own: torch.Tensor, k_buf: torch.Tensor, v_buf: torch.Tensor,
                out: torch.Tensor | None = None) -> torch.Tensor:
        """This rank's outputs [B,H,(s1-s0)*L,D].  q_own holds the rank's query frames; k_buf,
        v_buf are kv_buffers whose own part is filled (the halo part is overwritten)."""
        want = (self.s1 - self.h0) * self.L
        if k_buf.shape[2] != want or v_buf.shape[2] != want:
            raise ValueError(f"k/v buffers need {want} rows (halo + own frames)")
        if q_own.shape[2] != (self.s1 - self.s0) * self.L:
            raise ValueError("q_own must hold exactly this rank's frames")
        self._dims = rb.dims_of(q_own, self.Wq, self.P, self.phi)
        ws = self.workspace(q_own.device)
        kw = dict(T=self.T, c0=self.c0, c1=self.c1, P=self.P, phi=self.phi,
                  frame_tokens=self.L, Tc=self.Tc, To=self.To, workspace=ws)
        self._exchange_halo([k_buf, v_buf])
        S_seg, Z_seg = self.ops.segment_states(k_buf, v_buf, self.Wk, self.bk, **kw)
        S_all, Z_all = self._all_gather(S_seg), self._all_gather(Z_seg)
        S_pre = S_all[:self.rank].contiguous() if self.rank > 0 else None
        Z_pre = Z_all[:self.rank].contiguous() if self.rank > 0 else None
        return self.ops.segment_attend(q_own, k_buf, v_buf, self.Wq, self.bq, S_prefix=S_pre,
                                       Z_prefix=Z_pre, out=out, **kw)
