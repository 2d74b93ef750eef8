"""Head/batch sharding: the B*H independent (batch, head) problems of one forward split over the
ranks, each rank running the one-GPU library call on its share, the output slices all-gathered.

Nothing couples two (batch, head) pairs: the chunk recurrence of the "ReHyAt overview" page
(§2.3) runs along one head's token sequence, with that head's own feature-map weights.  So the
flattened units u = b*H + h are dealt out in contiguous ranges (`split_units`).  A rank's q, k, v
are a view of the full [B, H, N, D] tensors, presented to the library as one batch of n_r
"heads" ([1, n_r, N, D]), and its weights are its units' heads' weights gathered in unit order.
The library computes every unit the same way whatever other units share the call (the fold's
token splits depend on the sequence shape only), so the gathered output is bit-identical to the
one-call forward over all B*H units.

The process group must be initialised by the caller (NCCL for GPUs); every rank takes the same
collective steps in the same order.  The compute call comes from `ops` (the library binding by
default), so the host logic can be exercised with stand-in compute on CPU.
"""
from __future__ import annotations

import torch

from . import binding as rb


def split_units(n_units: int, world: int) -> list[tuple[int, int]]:
    """Contiguous unit ranges [u0, u1), one per rank, as even as possible (the first
    n_units % world ranks get one more).  Needs n_units >= world."""
    if world < 1 or n_units < world:
        raise ValueError(f"{n_units} (batch, head) units cannot be split over {world} ranks")
    base, extra = divmod(n_units, world)
    out, u0 = [], 0
    for r in range(world):
        u1 = u0 + base + (1 if r < extra else 0)
        out.append((u0, u1))
        u0 = u1
    return out


class HeadSharded:
    """The whole-sequence forward of B*H independent problems over the ranks of `group`."""

    def __init__(self, Wq, bq, Wk, bk, *, B: int, H: int, frame_tokens: int, Tc: int, To: int,
                 P: int, phi: int = rb.PHI_POLY, group=None, ops=None,
                 rank: int | None = None, world: int | None = None):
        """rank/world: plan as rank `rank` of `world` without a process group (one process
        running the ranks' shares one after another); `gather` is then unavailable."""
        import torch.distributed as dist
        self.dist = dist if dist.is_available() and dist.is_initialized() else None
        self.group = group
        if rank is not None or world is not None:
            self.dist = None
            self.rank, self.world = int(rank or 0), int(world or 1)
        else:
            self.rank = self.dist.get_rank(group) if self.dist else 0
            self.world = self.dist.get_world_size(group) if self.dist else 1
        self.ops = ops if ops is not None else rb
        self.B, self.H = B, H
        self.L, self.Tc, self.To, self.P, self.phi = frame_tokens, Tc, To, P, phi
        self.ranges = split_units(B * H, self.world)
        self.u0, self.u1 = self.ranges[self.rank]
        self.n_max = max(u1 - u0 for u0, u1 in self.ranges)
        heads = torch.tensor([u % H for u in range(self.u0, self.u1)], dtype=torch.long)
        idx = heads.to(Wq.device)
        # this rank's units' weights, in unit order (one "head" per unit)
        self.Wq = Wq.index_select(0, idx).contiguous()
        self.Wk = Wk.index_select(0, idx).contiguous()
        self.bq = bq.index_select(0, idx).contiguous() if bq is not None else None
        self.bk = bk.index_select(0, idx).contiguous() if bk is not None else None
        self._ws = None

    @property
    def n_units(self) -> int:
        return self.u1 - self.u0

    def shard(self, x: torch.Tensor) -> torch.Tensor:
        """This rank's units of a contiguous [B, H, N, D] tensor, as a [1, n_r, N, D] view."""
        if x.shape[:2] != (self.B, self.H) or not x.is_contiguous():
            raise ValueError(f"expected a contiguous [{self.B}, {self.H}, N, D] tensor")
        return x.view(1, self.B * self.H, *x.shape[2:])[:, self.u0:self.u1]

    def workspace(self, q_s: torch.Tensor) -> torch.Tensor:
        """The forward workspace of this rank's share (allocated once, reused)."""
        if self._ws is None or self._ws.device != q_s.device:
            d = rb.dims_of(q_s, self.Wq, self.P, self.phi)
            T = q_s.shape[2] // self.L
            n = self.ops.forward_workspace_size(d, rb._dtype_code(q_s), T, self.L, self.Tc,
                                                self.To)
            self._ws = torch.empty(max(n, 16), dtype=torch.uint8, device=q_s.device)
        return self._ws

    def forward(self, q_s: torch.Tensor, k_s: torch.Tensor, v_s: torch.Tensor,
                out: torch.Tensor | None = None) -> torch.Tensor:
        """This rank's outputs [1, n_r, N, D] from its shards (see `shard`)."""
        if q_s.shape[1] != self.n_units:
            raise ValueError(f"this rank holds {self.n_units} units, got {q_s.shape[1]}")
        return self.ops.forward(q_s, k_s, v_s, self.Wq, self.bq, self.Wk, self.bk, P=self.P,
                                phi=self.phi, frame_tokens=self.L, Tc=self.Tc, To=self.To,
                                workspace=self.workspace(q_s), out=out)

    def gather(self, out_s: torch.Tensor) -> torch.Tensor:
        """Every rank's output slice, assembled into [B, H, N, D] on every rank: one all-gather
        of equal-size slices (a rank with fewer units pads with zeros)."""
        N, D = out_s.shape[2], out_s.shape[3]
        if self.world == 1:
            return out_s.reshape(self.B, self.H, N, D)
        if self.dist is None:
            raise RuntimeError("gather needs the process group (this object plans one rank)")
        buf = out_s.new_zeros(1, self.n_max, N, D)
        buf[:, :self.n_units] = out_s
        parts = [torch.empty_like(buf) for _ in range(self.world)]
        self.dist.all_gather(parts, buf, group=self.group)
        full = torch.cat([p[:, :u1 - u0] for p, (u0, u1) in zip(parts, self.ranges)], dim=1)
        return full.reshape(self.B, self.H, N, D)
