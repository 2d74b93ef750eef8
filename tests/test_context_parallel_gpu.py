"""Context-parallel segments on one GPU: the ranks of a chunk-range split are emulated one after
another through the C ABI (each segment's states, then each segment's outputs from the sums of
the segments before it), with no kernel waiting on another.  Checked against the oracle on small
sequences and against the one-call forward (and sampled oracle rows at the segment boundaries)
at 480x832 5 s ("ReHyAt overview" §2.3: the state a chunk reads is the sum of all earlier
folds)."""
import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.context_parallel import split_chunks
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3


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


def run_segments(t, w: C.Workload, ranges):
    """Every segment's phase 1, then every segment's phase 2; returns the concatenated output."""
    q, k, v, Wq, bq, Wk, bk = t
    L = w.frame_tokens
    kw = dict(T=w.T, P=w.P, phi=w.phi_code, frame_tokens=L, Tc=w.Tc, To=w.To)
    d = rb.dims_of(q, Wq, w.P, w.phi_code)
    segs = []
    for (c0, c1) in ranges:
        s0, s1, h0 = rb.segment_bounds(w.T, w.Tc, w.To, c0, c1)
        k_seg = k[:, :, h0 * L:s1 * L].contiguous()
        v_seg = v[:, :, h0 * L:s1 * L].contiguous()
        ws = torch.empty(rb.segment_workspace_size(d, w.T, L, w.Tc, w.To, c0, c1),
                         dtype=torch.uint8, device=q.device)
        S, Z = rb.segment_states(k_seg, v_seg, Wk, bk, c0=c0, c1=c1, workspace=ws, **kw)
        segs.append((c0, c1, s0, s1, k_seg, v_seg, ws, S, Z))
    outs = []
    for r, (c0, c1, s0, s1, k_seg, v_seg, ws, _, _) in enumerate(segs):
        S_pre = torch.stack([sg[7] for sg in segs[:r]]) if r else None
        Z_pre = torch.stack([sg[8] for sg in segs[:r]]) if r else None
        out = torch.full_like(q[:, :, s0 * L:s1 * L], float("nan"))
        rb.segment_attend(q[:, :, s0 * L:s1 * L].contiguous(), k_seg, v_seg, Wq, bq, c0=c0,
                          c1=c1, workspace=ws, S_prefix=S_pre, Z_prefix=Z_pre, out=out, **kw)
        outs.append(out)
    return torch.cat(outs, dim=2)


def check(got, want, what):
    err, r = np.abs(got - want).max(), rel_l2(got, want)
    assert np.isfinite(got).all(), what + ": non-finite output"
    assert err <= BF16_MAX_ABS and r <= BF16_REL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {r:.3e}"


SMALL = [
    # T, frame h, w, Tc, To, P, ranks
    (13, 6, 11, 3, 1, 2, 2),
    (13, 6, 11, 3, 1, 2, 3),
    (13, 6, 11, 3, 1, 2, 5),     # one chunk per segment, the last ragged
    (14, 6, 11, 4, 2, 3, 2),     # wider halo, P = 3
    (12, 8, 16, 2, 3, 2, 3),     # To > Tc: halo frames reach two chunks back
]


@pytest.mark.parametrize("case", SMALL, ids=[f"T{c[0]}_Tc{c[3]}_To{c[4]}_R{c[6]}" for c in SMALL])
def test_segments_match_oracle(dev, case):
    T, fh, fw, Tc, To, P, R = case
    w = C.Workload("seg", B=1, H=2, D=128, T=T, frame_h=fh, frame_w=fw, Tc=Tc, To=To, P=P,
                   F=128, G=8, dtype="bf16", seed=41)
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    out = run_segments(t, w, split_chunks(w.n_chunks, R))
    rb.sync_status(dev)
    for h in range(2):
        q, k, v = f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h])
        want = O.hybrid_attention_quadratic(
            q, k, v, O.feature_map(q, f64(inp.Wq[h]), f64(inp.bq[h]), P),
            O.feature_map(k, f64(inp.Wk[h]), f64(inp.bk[h]), P), w.frame_tokens, Tc, To)
        check(f64(out[0, h]), want, f"R{R} h{h}")


def test_segment_sum_matches_closed_form(dev):
    """Phase 1's segment sum equals phi_k^T V over the frames the segment folds."""
    w = C.Workload("seg", B=1, H=2, D=128, T=13, frame_h=6, frame_w=11, Tc=3, To=1, P=2, F=128,
                   G=8, dtype="bf16", seed=43)
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    L = w.frame_tokens
    c0, c1 = 1, 3                      # folds of chunks 1 and 2: frames [2, 8)
    s0, s1, h0 = rb.segment_bounds(w.T, w.Tc, w.To, c0, c1)
    k_seg = t[1][:, :, h0 * L:s1 * L].contiguous()
    v_seg = t[2][:, :, h0 * L:s1 * L].contiguous()
    d = rb.dims_of(t[0], t[3], w.P)
    ws = torch.empty(rb.segment_workspace_size(d, w.T, L, w.Tc, w.To, c0, c1), dtype=torch.uint8,
                     device=dev)
    S, Z = rb.segment_states(k_seg, v_seg, t[5], t[6], T=w.T, c0=c0, c1=c1, P=w.P,
                             frame_tokens=L, Tc=w.Tc, To=w.To, workspace=ws)
    rb.sync_status(dev)
    for h in range(2):
        k, v = f64(inp.k[0, h])[2 * L:8 * L], f64(inp.v[0, h])[2 * L:8 * L]
        pk = O.feature_map(k, f64(inp.Wk[h]), f64(inp.bk[h]), w.P)
        S_want, Z_want = pk.T @ v, pk.sum(axis=0)
        assert rel_l2(f64(S[0, h]), S_want) <= 5e-3
        assert rel_l2(f64(Z[0, h]), Z_want) <= 5e-3


@pytest.mark.parametrize("R", [2, 4, 7])
def test_full_size_segments(dev, R):
    """480x832 5 s split over R emulated ranks: equals the one-call forward up to the order of
    the fp32 state sums, and sampled rows at every segment boundary match the oracle."""
    w = C.WAN_480P_5S
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    ranges = split_chunks(w.n_chunks, R)
    out = run_segments(t, w, ranges)
    ref = torch.full_like(t[0], float("nan"))
    rb.forward(*t, P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To, out=ref)
    rb.sync_status(dev)
    assert torch.isfinite(out).all()
    diff = (out.float() - ref.float())
    assert float(diff.abs().max()) <= 1e-2
    assert float(diff.norm() / ref.float().norm()) <= 1e-3
    L = w.frame_tokens
    rows = []
    for (c0, c1) in ranges:
        s0, s1, _ = rb.segment_bounds(w.T, w.Tc, w.To, c0, c1)
        rows += [s0 * L, s0 * L + 1, s0 * L + 200, s1 * L - 1]
    rows = np.array(sorted(set(rows)))
    for h in (0, 7):
        want = O.hybrid_attention_rows(f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h]),
                                       f64(inp.Wq[h]), f64(inp.bq[h]), f64(inp.Wk[h]),
                                       f64(inp.bk[h]), w.P, L, w.Tc, w.To, rows)
        check(f64(out[0, h][torch.as_tensor(rows, device=dev)]), want, f"R{R} h{h}")


def test_segment_argument_errors(dev):
    w = C.Workload("seg", B=1, H=1, D=128, T=6, frame_h=4, frame_w=4, Tc=2, To=1, P=2, F=128,
                   G=8, dtype="bf16", seed=1)
    d = rb.Dims(1, 1, 128, 128, 8, 2, 0)
    with pytest.raises(rb.RehyatError):
        rb.segment_workspace_size(d, w.T, w.frame_tokens, w.Tc, w.To, 2, 2)   # empty range
    with pytest.raises(rb.RehyatError):
        rb.segment_workspace_size(d, w.T, w.frame_tokens, w.Tc, w.To, 0, 4)   # past the end
