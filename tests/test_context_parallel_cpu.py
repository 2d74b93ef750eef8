"""Context parallelism's host path on CPU: gloo ranks (world size 2 and 3) run ContextParallel
with the oracle's float64 streaming step standing in for the library's segment calls, so the
chunk split, the halo exchange, the all-gather of the segment sums and their prefix order are
checked against the oracle's whole-sequence forward ("ReHyAt overview" §2.3: the state of a
chunk is the sum of all earlier folds)."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200.context_parallel import (ContextParallel, plan_ranks,
                                                                 split_chunks)
from oracle import rehyat_oracle as O

L, T, Tc, To, P = 6, 11, 2, 1, 2   # 6 chunks, the last one frame long
B, H, D, F, G = 1, 2, 16, 16, 4


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def make_data(seed=5):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, T * L, D, generator=g, dtype=torch.float64) for _ in range(3))
    Wq, Wk = (torch.randn(H, G, F // G, D // G, generator=g, dtype=torch.float64) * 0.5
              for _ in range(2))
    bq, bk = (torch.randn(H, F, generator=g, dtype=torch.float64) * 0.1 for _ in range(2))
    return q, k, v, Wq, bq, Wk, bk


class OracleOps:
    """The segment calls computed by the oracle (float64, CPU): the folds of the segment by
    their closed form, the outputs by the oracle's streaming step from the summed prefix."""

    def __init__(self, Wk, bk):
        self.Wk, self.bk = Wk, bk

    def segment_workspace_size(self, d, T_, L_, Tc_, To_, c0, c1):
        return 16

    def segment_states(self, k_seg, v_seg, Wk, bk, *, T, c0, c1, P, phi, frame_tokens, Tc, To,
                       workspace):
        C = math.ceil(T / Tc)
        s0, s1, h0 = rb.segment_bounds(T, Tc, To, c0, c1)
        end = min(c1, C - 1)
        wa = max(0, c0 * Tc - To)
        wb = max(0, end * Tc - To) if end > c0 else wa
        rows = slice((wa - h0) * frame_tokens, (wb - h0) * frame_tokens)
        S = torch.zeros(B, H, F, D, dtype=torch.float64)
        Z = torch.zeros(B, H, F, dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                kk = k_seg[b, h, rows].numpy()
                phi_k = O.feature_map(kk, Wk[h].numpy(), bk[h].numpy(), P)
                S[b, h] = torch.from_numpy(phi_k.T @ v_seg[b, h, rows].numpy())
                Z[b, h] = torch.from_numpy(phi_k.sum(axis=0))
        return S, Z

    def segment_attend(self, q_seg, k_seg, v_seg, Wq, bq, *, T, c0, c1, P, phi, frame_tokens,
                       Tc, To, workspace, S_prefix=None, Z_prefix=None, out=None):
        s0, s1, h0 = rb.segment_bounds(T, Tc, To, c0, c1)
        Lf = frame_tokens
        res = torch.empty(B, H, (s1 - s0) * Lf, D, dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                S = np.zeros((F, D)) if S_prefix is None else S_prefix[:, b, h].sum(0).numpy()
                Z = np.zeros(F) if Z_prefix is None else Z_prefix[:, b, h].sum(0).numpy()
                for c in range(c0, c1):
                    fs, fe = c * Tc, min((c + 1) * Tc, T)
                    o = min(To, fs)
                    win = slice((fs - o - h0) * Lf, (fe - h0) * Lf)
                    o_c, S, Z = O.chunk_forward(
                        q_seg[b, h, (fs - s0) * Lf:(fe - s0) * Lf].numpy(),
                        k_seg[b, h, win].numpy(), v_seg[b, h, win].numpy(), Wq[h].numpy(),
                        bq[h].numpy(), self.Wk[h].numpy(), self.bk[h].numpy(), P, S, Z, Lf, fs,
                        fe - fs, To)
                    res[b, h, (fs - s0) * Lf:(fe - s0) * Lf] = torch.from_numpy(o_c)
        return res


def expected():
    q, k, v, Wq, bq, Wk, bk = make_data()
    want = np.empty((B, H, T * L, D))
    for b in range(B):
        for h in range(H):
            qq, kk, vv = q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy()
            want[b, h] = O.hybrid_attention_quadratic(
                qq, kk, vv, O.feature_map(qq, Wq[h].numpy(), bq[h].numpy(), P),
                O.feature_map(kk, Wk[h].numpy(), bk[h].numpy(), P), L, Tc, To)
    return want


def _rank_main(rank, world, port, out_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, Wq, bq, Wk, bk = make_data()
        cp = ContextParallel(Wq, bq, Wk, bk, T=T, frame_tokens=L, Tc=Tc, To=To, P=P,
                             ops=OracleOps(Wk, bk))
        k_buf, v_buf = cp.kv_buffer(k).fill_(float("nan")), cp.kv_buffer(v).fill_(float("nan"))
        own = slice(cp.s0 * L, cp.s1 * L)
        cp.own(k_buf).copy_(k[:, :, own])
        cp.own(v_buf).copy_(v[:, :, own])
        out = cp.forward(q[:, :, own].contiguous(), k_buf, v_buf)
        # the halo really is the previous rank's frames
        halo = k[:, :, cp.h0 * L:cp.s0 * L]
        out_q.put((rank, cp.c0, cp.c1, out.numpy(), bool(torch.equal(k_buf[:, :, :halo.shape[2]],
                                                                     halo))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_matches_whole_sequence(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted((q.get(timeout=5) for _ in procs), key=lambda r: r[0])
    want = expected()
    covered = []
    for rank, c0, c1, out, halo_ok in res:
        s0, s1, _ = rb.segment_bounds(T, Tc, To, c0, c1)
        assert halo_ok
        got = out
        ref = want[:, :, s0 * L:s1 * L]
        assert np.abs(got - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
        covered.append((s0, s1))
    assert covered[0][0] == 0 and covered[-1][1] == T
    assert all(a[1] == b[0] for a, b in zip(covered, covered[1:]))


def test_single_process_is_one_segment():
    q, k, v, Wq, bq, Wk, bk = make_data()
    cp = ContextParallel(Wq, bq, Wk, bk, T=T, frame_tokens=L, Tc=Tc, To=To, P=P,
                         ops=OracleOps(Wk, bk))
    assert (cp.c0, cp.c1, cp.s0, cp.s1, cp.h0) == (0, 6, 0, T, 0)
    out = cp.forward(q, k.clone(), v.clone())
    np.testing.assert_allclose(out.numpy(), expected(), rtol=0, atol=1e-10)


def test_split_chunks():
    assert split_chunks(6, 2) == [(0, 3), (3, 6)]
    assert split_chunks(7, 3) == [(0, 3), (3, 5), (5, 7)]
    assert split_chunks(4, 4) == [(0, 1), (1, 2), (2, 3), (3, 4)]
    with pytest.raises(ValueError):
        split_chunks(2, 3)


def test_segment_bounds():
    # chunks [2, 4) of 11 frames, Tc = 2, To = 1: queries [4, 8), keys from frame 3
    assert rb.segment_bounds(11, 2, 1, 2, 4) == (4, 8, 3)
    assert rb.segment_bounds(11, 2, 1, 0, 2) == (0, 4, 0)
    assert rb.segment_bounds(11, 2, 3, 5, 6) == (10, 11, 7)   # ragged last chunk, wide halo


def test_plan_ranks():
    ranges, bounds = plan_ranks(11, 2, 1, 3)
    assert ranges == [(0, 2), (2, 4), (4, 6)]
    assert bounds == [(0, 4, 0), (4, 8, 3), (8, 11, 7)]
    # one frame per rank cannot supply a two-frame halo
    with pytest.raises(ValueError):
        plan_ranks(6, 1, 2, 6)
    # To wider than a chunk is fine while each rank holds enough frames
    ranges, bounds = plan_ranks(12, 2, 3, 3)
    assert bounds[1] == (4, 8, 1) and bounds[2] == (8, 12, 5)
