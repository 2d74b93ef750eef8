"""Host logic of the streaming session on CPU: the frame counter, the overlaps passed per step,
and checkpoint / resume, with the C call replaced by a host restatement of its carry contract
around the oracle's streaming step (the GPU path of the same session, where the library builds
the window, is covered by the gpu-marked tests)."""
import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import build
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200 import streaming
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs


@pytest.fixture
def oracle_step(monkeypatch):
    build.build()
    rb.load()
    calls = []

    def fake(q, k, v, Wq, bq, Wk, bk, S, Z, k_carry, v_carry, *, P, frame_tokens,
             frames_before, To, phi=0, To_next=None, out=None, workspace=None):
        """The carry contract of rehyat_chunk_forward_carry, restated on the host: window =
        [last min(To, frames_before) carried frames | chunk]; carry <- last cap frames of
        (carry ++ chunk), right-aligned; the step itself is the oracle's."""
        kind = O.PHI_ELU1 if phi == rb.PHI_ELU1 else O.PHI_POLY
        L = frame_tokens
        B, H, n, D = q.shape
        cf, cap = n // L, k_carry.shape[2] // L
        ov = min(To, frames_before)
        kw = torch.cat([k_carry[:, :, (cap - ov) * L:], k], dim=2)
        vw = torch.cat([v_carry[:, :, (cap - ov) * L:], v], dim=2)
        calls.append((frames_before, cf, kw.shape[2] // L))
        nxt = To if To_next is None else To_next
        out = torch.empty_like(q) if out is None else out
        for b in range(B):
            for h in range(H):
                o, Sn, Zn = O.chunk_forward(q[b, h].double().numpy(), kw[b, h].double().numpy(),
                                            vw[b, h].double().numpy(), Wq[h].double().numpy(),
                                            bq[h].double().numpy(), Wk[h].double().numpy(),
                                            bk[h].double().numpy(), P, S[b, h].double().numpy(),
                                            Z[b, h].double().numpy(), L, frames_before,
                                            cf, To, kind, To_next=nxt)
                out[b, h] = torch.from_numpy(o)
                S[b, h] = torch.from_numpy(Sn)
                Z[b, h] = torch.from_numpy(Zn)
        if cap:
            k_carry.copy_(torch.cat([k_carry, k], dim=2)[:, :, -cap * L:])
            v_carry.copy_(torch.cat([v_carry, v], dim=2)[:, :, -cap * L:])
        return out

    monkeypatch.setattr(streaming.rb, "chunk_forward_carry", fake)
    return calls


W = C.Workload("session-cpu", B=2, H=1, D=32, T=10, frame_h=2, frame_w=3, Tc=3, To=2, P=2, F=32,
               G=4, dtype="f32", seed=5)


def session():
    inp = make_inputs(W)
    s = streaming.ChunkStream(inp.Wq, inp.bq, inp.Wk, inp.bk, B=W.B, P=W.P,
                              frame_tokens=W.frame_tokens, Tc=W.Tc, To=W.To, dtype=torch.float32,
                              device=torch.device("cpu"))
    return inp, s


def feed(s, inp, chunks):
    L = W.frame_tokens
    return [s.step(inp.q[:, :, a * L:e * L].contiguous(), inp.k[:, :, a * L:e * L].contiguous(),
                   inp.v[:, :, a * L:e * L].contiguous()).clone() for (_, a, e) in chunks]


def test_windows_and_overlap(oracle_step):
    inp, s = session()
    out = torch.cat(feed(s, inp, W.chunk_bounds()), dim=2)
    # each call got the To frames before its chunk (fewer at the start) followed by the chunk
    assert oracle_step == [(0, 3, 3), (3, 3, 5), (6, 3, 5), (9, 1, 3)]
    for b in range(W.B):
        q, k, v = (x[b, 0].double().numpy() for x in (inp.q, inp.k, inp.v))
        want = O.hybrid_attention_quadratic(
            q, k, v, O.feature_map(q, inp.Wq[0].double().numpy(), inp.bq[0].double().numpy(), W.P),
            O.feature_map(k, inp.Wk[0].double().numpy(), inp.bk[0].double().numpy(), W.P),
            W.frame_tokens, W.Tc, W.To)
        got = out[b, 0].double().numpy()
        assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-6


def test_resume_from_host_state(oracle_step):
    inp, s = session()
    whole = feed(s, inp, W.chunk_bounds())
    inp, first = session()
    part1 = feed(first, inp, W.chunk_bounds()[:2])
    ck = first.state_dict()
    _, again = session()
    again.load_state_dict(ck)
    part2 = feed(again, inp, W.chunk_bounds()[2:])
    assert all(torch.equal(a, b) for a, b in zip(whole, part1 + part2))


def test_variable_schedule(oracle_step):
    """Longer first chunk and per-chunk overlaps (session capacity Tc = 4, To = 2)."""
    w = C.Workload("session-sched", B=1, H=1, D=32, T=11, frame_h=2, frame_w=2, Tc=4, To=2, P=2,
                   F=32, G=4, dtype="f32", seed=6)
    inp = make_inputs(w)
    cfs, ovs = [4, 2, 3, 1, 1], [0, 1, 2, 2, 0]
    s = streaming.ChunkStream(inp.Wq, inp.bq, inp.Wk, inp.bk, B=1, P=2, frame_tokens=4, Tc=4,
                              To=2, dtype=torch.float32, device=torch.device("cpu"))
    bounds = O.schedule_bounds(cfs, ovs)
    outs = []
    for c, (_, a, e) in enumerate(bounds):
        sl = slice(a * 4, e * 4)
        nxt = ovs[c + 1] if c + 1 < len(ovs) else ovs[c]
        outs.append(s.step(inp.q[:, :, sl].contiguous(), inp.k[:, :, sl].contiguous(),
                           inp.v[:, :, sl].contiguous(), To=ovs[c], To_next=nxt).clone())
    got = torch.cat(outs, dim=2)[0, 0].double().numpy()
    q, k, v = (x[0, 0].double().numpy() for x in (inp.q, inp.k, inp.v))
    pq = O.feature_map(q, inp.Wq[0].double().numpy(), inp.bq[0].double().numpy(), 2)
    pk = O.feature_map(k, inp.Wk[0].double().numpy(), inp.bk[0].double().numpy(), 2)
    want = O.hybrid_attention_masked(q, k, v, pq, pk, 4, O.schedule_mask(bounds))
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-6
    with pytest.raises(ValueError):
        s.step(inp.q[:, :, :4].contiguous(), inp.k[:, :, :4].contiguous(),
               inp.v[:, :, :4].contiguous(), To=3)
