"""The streaming session (ChunkStream): the sequence fed chunk by chunk with only S, Z and the
overlap frames carried matches the oracle, and a session checkpointed to host memory halfway
and resumed in a fresh session produces the same bits as the uninterrupted run."""
import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs
from hybrid_softmax_linear_chunked_b200.streaming import ChunkStream

pytestmark = pytest.mark.gpu

# 81 frames of 8 x 8 tokens, Tc = 3: 27 streaming calls, like the 20 s video at 480 x 832
W = C.Workload("stream-27", B=1, H=2, D=128, T=81, frame_h=8, frame_w=8, Tc=3, To=1, P=2, F=128,
               G=8, dtype="bf16", seed=31)


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_softmax_linear_chunked_b200 import build
    build.build()
    rb.load()
    return torch.device("cuda", 0)


@pytest.fixture(scope="module")
def data(dev):
    inp = make_inputs(W)
    return inp, [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]


def new_session(t, w=W):
    _, _, _, Wq, bq, Wk, bk = t
    return ChunkStream(Wq, bq, Wk, bk, B=w.B, P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc,
                       To=w.To)


def feed(sess, t, chunks, w=W):
    q, k, v = t[:3]
    L = w.frame_tokens
    outs = []
    for (_, s, e) in chunks:
        sl = slice(s * L, e * L)
        outs.append(sess.step(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                              v[:, :, sl].contiguous()).clone())
    return outs


def f64(x):
    return x.detach().to("cpu", torch.float64).numpy()


def test_session_matches_oracle(dev, data):
    inp, t = data
    sess = new_session(t)
    out = torch.cat(feed(sess, t, W.chunk_bounds()), dim=2)
    rb.sync_status(dev)
    for h in range(W.H):
        q, k, v = f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h])
        want = O.hybrid_attention_quadratic(q, k, v, O.feature_map(q, f64(inp.Wq[h]), f64(inp.bq[h]), W.P),
                                            O.feature_map(k, f64(inp.Wk[h]), f64(inp.bk[h]), W.P),
                                            W.frame_tokens, W.Tc, W.To)
        got = f64(out[0, h])
        assert np.isfinite(got).all()
        assert np.abs(got - want).max() <= 2e-2
        assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 5e-3
    assert sess.frames_seen == W.T


def test_checkpoint_resume_is_bit_identical(dev, data):
    _, t = data
    bounds = W.chunk_bounds()
    assert len(bounds) == 27
    whole = feed(new_session(t), t, bounds)

    first = new_session(t)
    part1 = feed(first, t, bounds[:13])
    ckpt = first.state_dict()
    assert ckpt["frames_seen"] == 39 and ckpt["S"].device.type == "cpu"
    del first
    torch.cuda.empty_cache()
    resumed = new_session(t)
    resumed.load_state_dict(ckpt)
    part2 = feed(resumed, t, bounds[13:])
    rb.sync_status(dev)
    for c, (a, b) in enumerate(zip(whole, part1 + part2)):
        assert torch.equal(a, b), f"chunk {c} differs after resume"


def test_ragged_last_chunk_and_wider_overlap(dev):
    """10 frames with Tc = 4 (last chunk 2 frames) and To = 2."""
    w = C.Workload("stream-ragged", B=2, H=1, D=128, T=10, frame_h=6, frame_w=11, Tc=4, To=2,
                   P=3, F=128, G=8, dtype="bf16", seed=33)
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    out = torch.cat(feed(new_session(t, w), t, w.chunk_bounds(), w), dim=2)
    rb.sync_status(dev)
    for b in range(2):
        q, k, v = f64(inp.q[b, 0]), f64(inp.k[b, 0]), f64(inp.v[b, 0])
        want = O.hybrid_attention_quadratic(q, k, v, O.feature_map(q, f64(inp.Wq[0]), f64(inp.bq[0]), w.P),
                                            O.feature_map(k, f64(inp.Wk[0]), f64(inp.bk[0]), w.P),
                                            w.frame_tokens, w.Tc, w.To)
        got = f64(out[b, 0])
        assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 5e-3


def test_session_rejects_bad_chunks_and_states(dev, data):
    _, t = data
    sess = new_session(t)
    q = t[0][:, :, :5 * W.frame_tokens].contiguous()   # 5 frames > Tc
    with pytest.raises(ValueError):
        sess.step(q, q, q)
    st = sess.state_dict()
    st["shape"] = (9,) + tuple(st["shape"][1:])
    with pytest.raises(ValueError):
        new_session(t).load_state_dict(st)


@pytest.mark.parametrize("cfs,ovs", [([5, 3, 3, 2], [0, 1, 2, 1]),
                                     # a 1-frame chunk under a 2-frame carry: the next carry
                                     # mixes carried and new frames
                                     ([3, 1, 2, 3], [0, 2, 2, 1])])
def test_variable_schedule(dev, cfs, ovs):
    """A longer first chunk and per-chunk overlaps (ReHyAt overview §5.2), bf16, against the
    quadratic form under the schedule's frame mask."""
    w = C.Workload("sched", B=1, H=2, D=128, T=sum(cfs), frame_h=6, frame_w=11, Tc=max(cfs),
                   To=max(ovs), P=2, F=128, G=8, dtype="bf16", seed=35)
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    q, k, v = t[:3]
    bounds = O.schedule_bounds(cfs, ovs)
    sess = new_session(t, w)
    L = w.frame_tokens
    outs = []
    for c, (_, s, e) in enumerate(bounds):
        sl = slice(s * L, e * L)
        nxt = ovs[c + 1] if c + 1 < len(ovs) else ovs[c]
        outs.append(sess.step(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                              v[:, :, sl].contiguous(), To=ovs[c], To_next=nxt).clone())
    rb.sync_status(dev)
    out = torch.cat(outs, dim=2)
    M = O.schedule_mask(bounds)
    for h in range(2):
        qh, kh, vh = f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h])
        want = O.hybrid_attention_masked(qh, kh, vh,
                                         O.feature_map(qh, f64(inp.Wq[h]), f64(inp.bq[h]), w.P),
                                         O.feature_map(kh, f64(inp.Wk[h]), f64(inp.bk[h]), w.P),
                                         L, M)
        got = f64(out[0, h])
        assert np.isfinite(got).all()
        assert np.abs(got - want).max() <= 2e-2
        assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 5e-3
