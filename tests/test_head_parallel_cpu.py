"""Head/batch sharding's host path on CPU: gloo ranks (world size 2, 3 and 5) each run
HeadSharded on their share of the B*H (batch, head) units, with the oracle's float64 forward
standing in for the library call, and all-gather the output slices.  The gathered result must
equal the oracle's forward over the whole problem exactly: each unit is computed from its own
head's weights, so a wrong unit range, a weight gathered from the wrong head or a slice put back
in the wrong place shows up ("ReHyAt overview" §2.3: the recurrence runs along one head's
sequence, so the (b, h) problems are independent)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from hybrid_softmax_linear_chunked_b200.head_parallel import HeadSharded, split_units
from oracle import rehyat_oracle as O

L, T, Tc, To, P = 5, 7, 3, 1, 2
B, H, D, F, G = 2, 3, 16, 16, 4


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def make_data(seed=7):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, T * L, D, generator=g) for _ in range(3))
    Wq, Wk = (torch.randn(H, G, F // G, D // G, generator=g) * 0.5 for _ in range(2))
    bq, bk = (torch.randn(H, F, generator=g) * 0.1 for _ in range(2))
    return q, k, v, Wq, bq, Wk, bk


def oracle_head(q, k, v, Wq, bq, Wk, bk):
    """One (b, h) problem by the oracle: q, k, v [N, D]; weights of that problem's head."""
    qq, kk, vv = (x.double().numpy() for x in (q, k, v))
    pq = O.feature_map(qq, Wq.double().numpy(), bq.double().numpy(), P)
    pk = O.feature_map(kk, Wk.double().numpy(), bk.double().numpy(), P)
    return O.hybrid_attention_quadratic(qq, kk, vv, pq, pk, L, Tc, To)


class OracleOps:
    """The library's whole-sequence forward computed by the oracle, head by head of the call."""

    def forward_workspace_size(self, d, code, T_, L_, Tc_, To_):
        return 16

    def forward(self, q, k, v, Wq, bq, Wk, bk, *, P, phi, frame_tokens, Tc, To, workspace,
                out=None):
        res = torch.empty(q.shape, dtype=torch.float64)
        for b in range(q.shape[0]):
            for h in range(q.shape[1]):
                res[b, h] = torch.from_numpy(oracle_head(q[b, h], k[b, h], v[b, h], Wq[h],
                                                         bq[h], Wk[h], bk[h]))
        return res


def expected():
    q, k, v, Wq, bq, Wk, bk = make_data()
    want = np.empty((B, H, T * L, D))
    for b in range(B):
        for h in range(H):
            want[b, h] = oracle_head(q[b, h], k[b, h], v[b, h], Wq[h], bq[h], Wk[h], bk[h])
    return want


def _rank_main(rank, world, port, out_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, Wq, bq, Wk, bk = make_data()
        hs = HeadSharded(Wq, bq, Wk, bk, B=B, H=H, frame_tokens=L, Tc=Tc, To=To, P=P,
                         ops=OracleOps())
        out_s = hs.forward(hs.shard(q), hs.shard(k), hs.shard(v))
        full = hs.gather(out_s)
        out_q.put((rank, hs.u0, hs.u1, full.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 5])
def test_head_sharded_matches_one_process(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    want = expected()
    ranges = split_units(B * H, world)
    for rank, u0, u1, full in res:
        assert (u0, u1) == ranges[rank]
        # every rank ends with the whole output, equal to the one-process oracle exactly
        np.testing.assert_array_equal(full, want)


def test_split_units():
    assert split_units(12, 8) == [(0, 2), (2, 4), (4, 6), (6, 8), (8, 9), (9, 10), (10, 11),
                                  (11, 12)]
    assert split_units(24, 1) == [(0, 24)]
    cover = [u for a, b in split_units(13, 4) for u in range(a, b)]
    assert cover == list(range(13))
    with pytest.raises(ValueError):
        split_units(3, 4)


def test_shard_views_and_weights():
    """One process planning rank 1 of 4 over B = 2, H = 3 (units 2, 3: (b0, h2) and (b1, h0)):
    its q is a view of the right rows and its weights are those units' heads."""
    q, k, v, Wq, bq, Wk, bk = make_data()
    hs = HeadSharded(Wq, bq, Wk, bk, B=B, H=H, frame_tokens=L, Tc=Tc, To=To, P=P,
                     ops=OracleOps(), rank=1, world=4)
    assert (hs.u0, hs.u1) == (2, 4)
    qs = hs.shard(q)
    assert qs.shape == (1, 2, T * L, D) and qs.data_ptr() == q[0, 2].data_ptr()
    assert torch.equal(qs[0, 1], q[1, 0])
    assert torch.equal(hs.Wq[0], Wq[2]) and torch.equal(hs.Wq[1], Wq[0])
    assert torch.equal(hs.bk[0], bk[2]) and torch.equal(hs.bk[1], bk[0])
    with pytest.raises(RuntimeError):
        hs.gather(hs.forward(qs, hs.shard(k), hs.shard(v)))
