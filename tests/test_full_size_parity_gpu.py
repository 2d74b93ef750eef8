"""Full-size parity of the CUDA path with the float64 oracle: every row of selected heads, bounds
asserted chunk by chunk, and pins that isolate the windowed softmax at full size.

With the workloads' random feature-map weights the linear branch carries tens to hundreds of
times the softmax branch's mass in every chunk after the first, so an error in the windowed
softmax of those chunks is divided by that factor before it reaches a whole-output tolerance.
Two things close that gap:

* the bounds (max-abs <= 2e-2 and relative L2 <= 5e-3, bf16 inputs with fp32 accumulation) hold
  for every chunk's rows on their own, not only for the whole output;
* a bias of -30 in both feature maps makes phi ~ e^(u - 30): the linear mass falls below 1e-18 of
  the softmax mass and the output is the plain softmax over each chunk's window (the output
  formula of the "ReHyAt overview" page, §2.2.1, with nothing left in the linear region).  Torch's
  float64 scaled_dot_product_attention computes that chunk by chunk from the window alone, with
  no mask and independently of the oracle.  At 1560- and 3600-token frames a window is 37-113 key
  tiles long, so the long-window rescaling, the grid order and the ragged last tiles of the
  attention kernel are all on the path.

Every output buffer starts as NaN, so a row the kernels never write fails the finiteness check.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3
WINDOW_ONLY_BIAS = -30.0


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_softmax_linear_chunked_b200 import build
    build.build()
    rb.load()
    return torch.device("cuda", 0)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def check_by_chunk(got, want, w: C.Workload, what: str, rows=None):
    """Bounds on every chunk's rows and on the whole.  got/want: [n, D]; `rows` are the query row
    indices of the n rows (default: all rows of the sequence, in order)."""
    rows = np.arange(len(got)) if rows is None else np.asarray(rows)
    chunk = rows // w.frame_tokens // w.Tc
    assert np.isfinite(got).all(), f"{what}: non-finite (unwritten) output rows"
    lines, bad = [], []
    for c in np.unique(chunk):
        sel = chunk == c
        a, b = got[sel], want[sel]
        err, r = float(np.abs(a - b).max()), rel_l2(a, b)
        lines.append(f"c{c}: {r:.1e}/{err:.1e}")
        if err > MAX_ABS or r > REL_L2:
            bad.append(int(c))
    err, r = float(np.abs(got - want).max()), rel_l2(got, want)
    msg = (f"{what}: max-abs {err:.3e}, rel-L2 {r:.3e}; per chunk (rel-L2/max-abs) "
           + " ".join(lines))
    assert not bad and err <= MAX_ABS and r <= REL_L2, f"chunks {bad} out of bounds. " + msg
    return msg


def run_forward(inp, w, dev):
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    out = torch.full_like(q, float("nan"))
    rb.forward(q, k, v, Wq, bq, Wk, bk, P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To,
               out=out)
    rb.sync_status(dev)
    return out


def oracle_recurrent(inp, w, b, h):
    q, k, v = f64(inp.q[b, h]), f64(inp.k[b, h]), f64(inp.v[b, h])
    pq = O.feature_map(q, f64(inp.Wq[h]), f64(inp.bq[h]), w.P)
    pk = O.feature_map(k, f64(inp.Wk[h]), f64(inp.bk[h]), w.P)
    return O.hybrid_attention_recurrent(q, k, v, pq, pk, w.frame_tokens, w.Tc, w.To)


def windowed_softmax_sdpa(inp, w, b, h, bounds=None):
    """Softmax over each chunk's window, chunk by chunk, by torch's float64 SDPA (no mask: the
    window of chunk c is exactly the keys of frames [w_c, e_c))."""
    L = w.frame_tokens
    q, k, v = (x[b, h].double() for x in (inp.q, inp.k, inp.v))
    out = torch.empty_like(q)
    for (wf, s, e) in (bounds or w.chunk_bounds()):
        out[s * L:e * L] = torch.nn.functional.scaled_dot_product_attention(
            q[None, s * L:e * L], k[None, wf * L:e * L], v[None, wf * L:e * L])[0]
    return out.numpy()


def sample_rows(w: C.Workload, n_per_chunk: int, rng):
    """Random rows of every chunk plus the rows at its first two tile boundaries and its end."""
    L = w.frame_tokens
    rows = []
    for (_, s, e) in w.chunk_bounds():
        lo, hi = s * L, e * L
        pick = {lo, lo + 127, lo + 128, hi - 1, min(hi - 1, lo + 255), min(hi - 1, lo + 256)}
        pick |= set(int(x) for x in rng.integers(lo, hi, size=n_per_chunk))
        rows.extend(sorted(pick))
    return np.array(rows)


def oracle_rows(inp, w, b, h, rows):
    return O.hybrid_attention_rows(f64(inp.q[b, h]), f64(inp.k[b, h]), f64(inp.v[b, h]),
                                   f64(inp.Wq[h]), f64(inp.bq[h]), f64(inp.Wk[h]),
                                   f64(inp.bk[h]), w.P, w.frame_tokens, w.Tc, w.To, rows)


FULL = [C.WAN_480P_5S, C.WAN_480P_10S, C.WAN_720P_5S]
FULL_IDS = ["480p5s", "480p10s", "720p5s"]


@pytest.mark.parametrize("w", FULL, ids=FULL_IDS)
def test_every_row_two_heads(dev, w):
    """Every query row of the first and the last head against the oracle's recurrent form (itself
    pinned equal to the quadratic form), chunk by chunk."""
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    assert torch.isfinite(out).all(), "output has unwritten (NaN) or non-finite rows"
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        print(check_by_chunk(f64(out[b, h]), oracle_recurrent(inp, w, b, h), w,
                             f"{w.name} b{b} h{h}"))


@pytest.mark.parametrize("w", FULL, ids=FULL_IDS)
def test_windowed_softmax_full_size(dev, w):
    """bias -30: the output is the softmax over each chunk's window.  Every row of two heads
    against float64 SDPA per window, and sampled rows of every head against the oracle."""
    w = dataclasses.replace(w, bias=WINDOW_ONLY_BIAS, name=w.name + ", bias -30")
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    assert torch.isfinite(out).all(), "output has unwritten (NaN) or non-finite rows"
    for (b, h) in [(0, 1), (w.B - 1, w.H - 2)]:
        print(check_by_chunk(f64(out[b, h]), windowed_softmax_sdpa(inp, w, b, h), w,
                             f"{w.name} b{b} h{h} vs SDPA"))
    rows = sample_rows(w, 4, np.random.default_rng(3))
    idx = torch.as_tensor(rows, device=out.device)
    for h in range(w.H):
        check_by_chunk(f64(out[0, h][idx]), oracle_rows(inp, w, 0, h, rows), w,
                       f"{w.name} b0 h{h} sampled vs oracle", rows=rows)


def stream_session(inp, w, dev):
    """The workload fed chunk by chunk through the streaming session (the library reads each
    window from its carried frames and the new chunk); returns the output and the peak device
    memory after every call."""
    from hybrid_softmax_linear_chunked_b200.streaming import ChunkStream
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    L = w.frame_tokens
    sess = ChunkStream(Wq, bq, Wk, bk, B=w.B, P=w.P, frame_tokens=L, Tc=w.Tc, To=w.To)
    chunks = [[x[:, :, s * L:e * L].contiguous() for x in (q, k, v)]
              for (_, s, e) in w.chunk_bounds()]
    outs = [torch.full_like(c[0], float("nan")) for c in chunks]
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    mem = []
    for c, (qc, kc, vc) in enumerate(chunks):
        sess.step(qc, kc, vc, out=outs[c])
        mem.append(torch.cuda.max_memory_allocated(dev))
    rb.sync_status(dev)
    return torch.cat(outs, dim=2), mem


def test_streaming_session_20s_windowed_softmax(dev):
    """480x832 20 s, B = 2, through the streaming session with bias -30: each window is read from
    two segments (the carried 1560-token frame and the new chunk), each with a ragged last tile.
    Every row of two (b, h) against float64 SDPA per window; constant device memory."""
    w = dataclasses.replace(C.WAN_480P_20S_STREAM, bias=WINDOW_ONLY_BIAS)
    inp = make_inputs(w)
    out, mem = stream_session(inp, w, dev)
    assert torch.isfinite(out).all()
    assert len(set(mem)) == 1, f"peak device memory grew across chunks: {mem}"
    for (b, h) in [(0, 2), (1, 9)]:
        print(check_by_chunk(f64(out[b, h]), windowed_softmax_sdpa(inp, w, b, h), w,
                             f"20 s stream, bias -30, b{b} h{h} vs SDPA"))


def test_streaming_session_20s_every_row(dev):
    """480x832 20 s through the streaming session with the standard inputs: every row of one
    (b, h) against the oracle's recurrent form, so the state carried over 27 calls is checked
    in every chunk."""
    w = C.WAN_480P_20S_STREAM
    inp = make_inputs(w)
    out, mem = stream_session(inp, w, dev)
    assert len(set(mem)) == 1, f"peak device memory grew across chunks: {mem}"
    print(check_by_chunk(f64(out[1, 11]), oracle_recurrent(inp, w, 1, 11), w,
                         "20 s stream b1 h11"))


ABLATION = [(tc, to, p) for tc in (1, 3, 5) for to in (0, 1) for p in (1, 2, 3)]
ABLATION += [(3, 2, 2), (5, 2, 2)]  # the wider overlap (To = 2) the pages also discuss


@pytest.mark.parametrize("Tc,To,P", ABLATION, ids=[f"Tc{a}_To{b}_P{c}" for a, b, c in ABLATION])
def test_ablation_sweep(dev, Tc, To, P):
    """The 21-frame 480x832 shape at every point of the Tc x To x P sweep (+ To = 2): four heads,
    every row of two of them against the recurrent oracle and sampled rows of the other two
    against the row oracle, chunk by chunk."""
    w = C.ablation(Tc, To, P)
    inp = make_inputs(w, heads=4)
    out = run_forward(inp, w, dev)
    assert torch.isfinite(out).all()
    for h in (0, 3):
        check_by_chunk(f64(out[0, h]), oracle_recurrent(inp, w, 0, h), w, f"{w.name} h{h}")
    rows = sample_rows(w, 3, np.random.default_rng(Tc * 100 + To * 10 + P))
    idx = torch.as_tensor(rows, device=out.device)
    for h in (1, 2):
        check_by_chunk(f64(out[0, h][idx]), oracle_rows(inp, w, 0, h, rows), w,
                       f"{w.name} h{h} sampled", rows=rows)
