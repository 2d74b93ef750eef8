"""Parity of the CUDA path (through the C ABI) with the float64 oracle, on seeded inputs.

Tolerances: bf16 inputs with fp32 accumulation -> max-abs <= 2e-2 and relative L2 <= 5e-3;
fp32 inputs -> relative L2 <= 1e-5.  Outputs are poisoned with NaN before every call so that a
row the kernels fail to write shows up.
"""
import math

import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_REL_L2 = 1e-5


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_softmax_linear_chunked_b200 import build
    build.build()
    rb.load()
    return torch.device("cuda", 0)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def to_dev(inp, dev):
    return [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]


def oracle_head(inp, b, h, w: C.Workload):
    q, k, v = f64(inp.q[b, h]), f64(inp.k[b, h]), f64(inp.v[b, h])
    pq = O.feature_map(q, f64(inp.Wq[h]), f64(inp.bq[h]), w.P)
    pk = O.feature_map(k, f64(inp.Wk[h]), f64(inp.bk[h]), w.P)
    return O.hybrid_attention_quadratic(q, k, v, pq, pk, w.frame_tokens, w.Tc, w.To)


def run_forward(inp, w, dev):
    q, k, v, Wq, bq, Wk, bk = to_dev(inp, dev)
    out = torch.full_like(q, float("nan"))
    rb.forward(q, k, v, Wq, bq, Wk, bk, P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To,
               out=out)
    rb.sync_status(dev)
    return out


def check_bf16(got, want, what, per_chunk_L=None, Tc=None):
    err = np.abs(got - want).max()
    r = rel_l2(got, want)
    msg = f"{what}: max-abs {err:.3e}, rel-L2 {r:.3e}"
    if per_chunk_L:
        rows = Tc * per_chunk_L
        parts = [f"{rel_l2(got[i:i + rows], want[i:i + rows]):.1e}" for i in range(0, len(got), rows)]
        msg += " per chunk " + " ".join(parts)
    assert np.isfinite(got).all(), what + ": non-finite output"
    assert err <= BF16_MAX_ABS and r <= BF16_REL_L2, msg
    return msg


# ------------------------------------------------------------------------------------------
# feature map
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("P,G", [(2, 8), (3, 8), (1, 4), (2, 16)])
def test_featmap_bf16(dev, P, G):
    w = C.Workload("fm", B=2, H=3, D=128, T=1, frame_h=1, frame_w=300, Tc=1, To=0, P=P, F=128,
                   G=G, dtype="bf16", bias=0.3, seed=11)
    inp = make_inputs(w)
    phi = rb.featmap(inp.q.to(dev), inp.Wq.to(dev), inp.bq.to(dev), P)
    for b in range(2):
        for h in range(3):
            want = O.feature_map(f64(inp.q[b, h]), f64(inp.Wq[h]), f64(inp.bq[h]), P)
            got = f64(phi[b, h])
            np.testing.assert_allclose(got, want, rtol=8e-3, atol=1e-6)


def test_featmap_f32(dev):
    w = C.TINY_F32
    inp = make_inputs(w)
    phi = rb.featmap(inp.q.to(dev), inp.Wq.to(dev), inp.bq.to(dev), w.P)
    want = O.feature_map(f64(inp.q[0, 0]), f64(inp.Wq[0]), f64(inp.bq[0]), w.P)
    np.testing.assert_allclose(f64(phi[0, 0]), want, rtol=2e-6, atol=1e-7)


# ------------------------------------------------------------------------------------------
# fp32 path: the tiny workload
# ------------------------------------------------------------------------------------------

def test_tiny_f32_forward(dev):
    w = C.TINY_F32
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    want = oracle_head(inp, 0, 0, w)
    assert rel_l2(f64(out[0, 0]), want) <= F32_REL_L2


def test_tiny_f32_bruteforce(dev):
    """The same output against the scalar brute force (independent of the quadratic form)."""
    w = C.TINY_F32
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    want = O.hybrid_attention_bruteforce(f64(inp.q[0, 0]), f64(inp.k[0, 0]), f64(inp.v[0, 0]),
                                         f64(inp.Wq[0]), f64(inp.bq[0]), f64(inp.Wk[0]),
                                         f64(inp.bk[0]), w.P, w.frame_tokens, w.Tc, w.To)
    assert rel_l2(f64(out[0, 0]), want) <= F32_REL_L2


@pytest.mark.parametrize("Tc,To,P", [(1, 0, 1), (2, 3, 3), (4, 1, 2)])
def test_f32_schedules(dev, Tc, To, P):
    w = C.Workload("f32 sched", B=2, H=2, D=64, T=9, frame_h=3, frame_w=7, Tc=Tc, To=To, P=P,
                   F=48, G=4, dtype="f32", seed=3)
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    for b in range(2):
        for h in range(2):
            assert rel_l2(f64(out[b, h]), oracle_head(inp, b, h, w)) <= F32_REL_L2


def stream(inp, w, dev, check_states=True):
    """Feed the sequence chunk by chunk through chunk_forward (only S, Z and the overlap frames
    carried between calls); return outputs, the states after each call, and the peak device
    memory after each call (every buffer is allocated before the loop)."""
    q, k, v, Wq, bq, Wk, bk = to_dev(inp, dev)
    B, H, N, D = q.shape
    L = w.frame_tokens
    bounds = w.chunk_bounds()
    S = torch.zeros(B, H, w.F, D, dtype=torch.float32, device=dev)
    Z = torch.zeros(B, H, w.F, dtype=torch.float32, device=dev)
    outs = [torch.full((B, H, (e - s) * L, D), float("nan"), dtype=q.dtype, device=dev)
            for (_, s, e) in bounds]
    states = [(torch.empty_like(S), torch.empty_like(Z)) for _ in bounds] if check_states else []
    ws = torch.empty(rb.chunk_workspace_size(rb.dims_of(q, Wq, w.P), rb._dtype_code(q), L, w.Tc,
                                             w.To), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    peaks = []
    for c, (wf, s, e) in enumerate(bounds):
        qc = q[:, :, s * L:e * L].contiguous()
        kw = k[:, :, wf * L:e * L].contiguous()
        vw = v[:, :, wf * L:e * L].contiguous()
        rb.chunk_forward(qc, kw, vw, Wq, bq, Wk, bk, S, Z, P=w.P, frame_tokens=L,
                         frames_before=s, To=w.To, out=outs[c], workspace=ws)
        del qc, kw, vw
        if check_states:
            states[c][0].copy_(S)
            states[c][1].copy_(Z)
        peaks.append(torch.cuda.max_memory_allocated(dev))
    rb.sync_status(dev)
    return torch.cat(outs, dim=2), states, peaks


def test_tiny_f32_streaming(dev):
    w = C.TINY_F32
    inp = make_inputs(w)
    out, states, _ = stream(inp, w, dev)
    want = oracle_head(inp, 0, 0, w)
    assert rel_l2(f64(out[0, 0]), want) <= F32_REL_L2
    # the state after the last chunk holds every frame before T - To
    k, v = f64(inp.k[0, 0]), f64(inp.v[0, 0])
    pk = O.feature_map(k, f64(inp.Wk[0]), f64(inp.bk[0]), w.P)
    m = (w.T - w.To) * w.frame_tokens
    S, Z = states[-1]
    assert rel_l2(f64(S[0, 0]), pk[:m].T @ v[:m]) <= 1e-6
    assert rel_l2(f64(Z[0, 0]), pk[:m].sum(0)) <= 1e-6


# ------------------------------------------------------------------------------------------
# bf16 path, sizes the oracle evaluates whole
# ------------------------------------------------------------------------------------------

SMALL = [
    # (T, frame_h, frame_w, Tc, To, P, G, B, H, k_scale, bias)
    (7, 10, 20, 3, 1, 2, 8, 1, 2, 1.0, 0.0),    # 200-token frames: ragged tiles, 3 chunks
    (5, 10, 13, 1, 0, 1, 8, 2, 1, 1.0, 0.0),    # Tc = 1, To = 0
    (8, 8, 12, 5, 2, 3, 8, 1, 2, 1.0, 0.0),     # Tc = 5, To = 2, P = 3, ragged last chunk
    (4, 8, 8, 4, 1, 2, 8, 1, 1, 1.0, 0.0),      # one chunk: plain softmax attention
    (9, 1, 17, 2, 3, 2, 4, 1, 2, 2.0, 0.0),     # 17-token frames, To > Tc, k x 2, G = 4
    (6, 16, 16, 3, 1, 2, 16, 1, 1, 1.0, 0.0),   # 256-token frames (tile-aligned), G = 16
    (6, 8, 16, 2, 1, 2, 2, 1, 1, 1.0, 0.0),     # G = 2 (wide groups)
    (5, 8, 16, 2, 1, 2, 1, 1, 1, 1.0, 0.0),     # G = 1 (dense 1x1 linear)
    (7, 10, 20, 3, 1, 2, 8, 1, 1, 1.0, -30.0),  # bias -30: linear mass ~1e-18, windowed softmax
    (7, 10, 20, 3, 1, 2, 8, 1, 1, 1.0, 4.0),    # bias +4: linear term dominates
]


@pytest.mark.parametrize("case", SMALL, ids=[f"T{c[0]}_L{c[1]*c[2]}_Tc{c[3]}_To{c[4]}_P{c[5]}_G{c[6]}_k{c[9]}_b{c[10]}" for c in SMALL])
def test_bf16_forward_small(dev, case):
    T, fh, fw, Tc, To, P, G, B, H, ks, bias = case
    w = C.Workload("small", B=B, H=H, D=128, T=T, frame_h=fh, frame_w=fw, Tc=Tc, To=To, P=P,
                   F=128, G=G, dtype="bf16", k_scale=ks, bias=bias, seed=5)
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    for b in range(B):
        for h in range(H):
            check_bf16(f64(out[b, h]), oracle_head(inp, b, h, w), f"b{b} h{h}",
                       per_chunk_L=w.frame_tokens, Tc=Tc)


def test_bf16_windowed_softmax_pin(dev):
    """bias = -30 makes the linear branch vanish: the output is softmax over each chunk's window,
    which torch's float64 scaled_dot_product_attention computes with a block mask."""
    w = C.Workload("win", B=1, H=1, D=128, T=7, frame_h=10, frame_w=20, Tc=3, To=1, P=2, F=128,
                   G=8, dtype="bf16", bias=-30.0, seed=9)
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    L, N = w.frame_tokens, w.N
    mask = torch.zeros(N, N, dtype=torch.bool)
    for (wf, s, e) in w.chunk_bounds():
        mask[s * L:e * L, wf * L:e * L] = True
    q, k, v = (x[0, 0].double() for x in (inp.q, inp.k, inp.v))
    want = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None],
                                                            attn_mask=mask[None])[0].numpy()
    check_bf16(f64(out[0, 0]), want, "windowed softmax")


def test_bf16_chunk_states(dev):
    w = C.Workload("states", B=1, H=2, D=128, T=8, frame_h=10, frame_w=20, Tc=3, To=1, P=2,
                   F=128, G=8, dtype="bf16", seed=4)
    inp = make_inputs(w)
    _, k, v, _, _, Wk, bk = to_dev(inp, dev)
    S, Z = rb.chunk_states(k, v, Wk, bk, P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To)
    rb.sync_status(dev)
    for h in range(2):
        Sw, Zw = O.prefix_states(f64(inp.k[0, h]), f64(inp.v[0, h]), f64(inp.Wk[h]),
                                 f64(inp.bk[h]), w.P, w.frame_tokens, w.Tc, w.To)
        for c in range(w.n_chunks):
            if c == 0:
                assert np.abs(f64(S[0, h, 0])).max() == 0 and np.abs(f64(Z[0, h, 0])).max() == 0
                continue
            assert rel_l2(f64(S[0, h, c]), Sw[c]) <= 5e-3, f"S chunk {c}"
            assert rel_l2(f64(Z[0, h, c]), Zw[c]) <= 5e-3, f"Z chunk {c}"


def test_bf16_streaming_small(dev):
    w = C.Workload("stream", B=1, H=2, D=128, T=10, frame_h=10, frame_w=13, Tc=3, To=1, P=2,
                   F=128, G=8, dtype="bf16", seed=8)
    inp = make_inputs(w)
    out, states, mem = stream(inp, w, dev)
    L = w.frame_tokens
    for h in range(2):
        check_bf16(f64(out[0, h]), oracle_head(inp, 0, h, w), f"stream h{h}", per_chunk_L=L,
                   Tc=w.Tc)
        pk = O.feature_map(f64(inp.k[0, h]), f64(inp.Wk[h]), f64(inp.bk[h]), w.P)
        v = f64(inp.v[0, h])
        for c, (wf, s, e) in enumerate(w.chunk_bounds()):
            m = max(0, e - w.To) * L
            S, Z = states[c]
            assert rel_l2(f64(S[0, h]), pk[:m].T @ v[:m]) <= 5e-3
            assert rel_l2(f64(Z[0, h]), pk[:m].sum(0)) <= 5e-3
    assert len(set(mem[1:])) == 1, f"peak device memory grew across chunks: {mem}"


def test_streaming_matches_forward_bf16(dev):
    """The streaming calls and the whole-sequence call compute the same outputs."""
    w = C.Workload("stream-vs-full", B=1, H=2, D=128, T=9, frame_h=12, frame_w=12, Tc=3, To=1,
                   P=2, F=128, G=8, dtype="bf16", seed=12)
    inp = make_inputs(w)
    full = run_forward(inp, w, dev)
    st, _, _ = stream(inp, w, dev, check_states=False)
    a, b = f64(st), f64(full)
    assert rel_l2(a, b) <= 3e-3 and np.abs(a - b).max() <= 1e-2


# ------------------------------------------------------------------------------------------
# full-size workloads: sampled rows against the oracle evaluated row by row
# ------------------------------------------------------------------------------------------

def sample_rows(w: C.Workload, n_per_chunk: int, rng):
    L = w.frame_tokens
    rows = []
    for (wf, s, e) in w.chunk_bounds():
        lo, hi = s * L, e * L
        pick = {lo, lo + 127, lo + 128, hi - 1, min(hi - 1, lo + 255), min(hi - 1, lo + 256)}
        pick |= set(int(x) for x in rng.integers(lo, hi, size=n_per_chunk))
        rows.extend(sorted(pick))
    return np.array(rows)


def check_sampled(out, inp, w, rows, heads):
    worst = 0.0
    for (b, h) in heads:
        want = O.hybrid_attention_rows(f64(inp.q[b, h]), f64(inp.k[b, h]), f64(inp.v[b, h]),
                                       f64(inp.Wq[h]), f64(inp.bq[h]), f64(inp.Wk[h]),
                                       f64(inp.bk[h]), w.P, w.frame_tokens, w.Tc, w.To, rows)
        got = f64(out[b, h][torch.as_tensor(rows, device=out.device)])
        check_bf16(got, want, f"{w.name} b{b} h{h}")
        worst = max(worst, rel_l2(got, want))
    return worst


@pytest.mark.parametrize("w", [C.WAN_480P_5S, C.WAN_480P_10S, C.WAN_720P_5S],
                         ids=["480p5s", "480p10s", "720p5s"])
def test_full_size_sampled(dev, w):
    inp = make_inputs(w)
    out = run_forward(inp, w, dev)
    assert torch.isfinite(out).all(), "output has unwritten (NaN) or non-finite rows"
    rng = np.random.default_rng(0)
    rows = sample_rows(w, 6, rng)
    heads = [(0, h) for h in range(w.H)]
    check_sampled(out, inp, w, rows, heads)


def test_full_size_streaming_20s(dev):
    """480x832 20 s, B = 2, fed chunk by chunk: sampled rows of every chunk against the oracle,
    and constant device memory across the 27 calls."""
    w = C.WAN_480P_20S_STREAM
    inp = make_inputs(w)
    out, _, mem = stream(inp, w, dev, check_states=False)
    assert torch.isfinite(out).all()
    assert len(set(mem[1:])) == 1, f"peak device memory grew across chunks: {mem}"
    print(f"peak device memory after chunks 3, 9, 27: {mem[2]}, {mem[8]}, {mem[26]} bytes")
    rng = np.random.default_rng(1)
    rows = sample_rows(w, 2, rng)
    check_sampled(out, inp, w, rows, [(0, 0), (1, 7), (1, 11)])


def test_full_size_streaming_session_20s(dev):
    """The same workload through the streaming session (the library assembles each window from
    the carried frames): sampled rows against the oracle, constant device memory, and the same
    outputs as the window-slicing loop above up to accumulation order."""
    from hybrid_softmax_linear_chunked_b200.streaming import ChunkStream
    w = C.WAN_480P_20S_STREAM
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = to_dev(inp, dev)
    L = w.frame_tokens
    sess = ChunkStream(Wq, bq, Wk, bk, B=w.B, P=w.P, frame_tokens=L, Tc=w.Tc, To=w.To)
    bounds = w.chunk_bounds()
    chunks = [[x[:, :, s * L:e * L].contiguous() for x in (q, k, v)] for (_, s, e) in bounds]
    outs = [torch.full_like(c[0], float("nan")) for c in chunks]
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    mem = []
    for c, (qc, kc, vc) in enumerate(chunks):
        sess.step(qc, kc, vc, out=outs[c])
        mem.append(torch.cuda.max_memory_allocated(dev))
    rb.sync_status(dev)
    out = torch.cat(outs, dim=2)
    assert torch.isfinite(out).all()
    assert len(set(mem)) == 1, f"peak device memory grew across chunks: {mem}"
    rng = np.random.default_rng(2)
    rows = sample_rows(w, 2, rng)
    check_sampled(out, inp, w, rows, [(0, 3), (1, 5)])


# ------------------------------------------------------------------------------------------
# argument errors reported through the C ABI with a GPU present
# ------------------------------------------------------------------------------------------

def test_errors_reported(dev):
    w = C.Workload("err", B=1, H=1, D=64, T=3, frame_h=4, frame_w=4, Tc=1, To=0, P=2, F=64,
                   G=8, dtype="bf16")
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = to_dev(inp, dev)
    with pytest.raises(rb.RehyatError) as e:
        rb.forward(q, k, v, Wq, bq, Wk, bk, P=2, frame_tokens=16, Tc=1, To=0)
    assert e.value.status == -2  # D = 64 is not a bf16-path shape
