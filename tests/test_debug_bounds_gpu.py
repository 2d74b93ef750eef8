"""The debug-bounds build (REHYAT_DEBUG_BOUNDS): every TMA coordinate and global store index of the
forward kernels is checked, and a failed check is reported through rehyat_sync_status as
REHYAT_ERR_BOUNDS instead of faulting.

* No false positives: the whole-sequence forward, the streaming step on carried frames (two-segment
  windows, a lone last tile split into parts) and the segment calls run through the checking
  build, match the oracle and leave the error word clear; so does the backward (its TMA
  reduce-adds are checked), whose gradients match the normal build's.
* The check fires: the self test's out-of-range store (into slack the test allocated, so the
  write would stay inside the buffer even without the check) is recorded and skipped.
The normal library is restored for the tests that follow."""
import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import build
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    normal = build.build()
    lib = rb.use_library(build.build(debug_bounds=True))
    assert lib.rehyat_debug_bounds() == 1
    yield torch.device("cuda", 0)
    rb.use_library(normal)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check(got, want):
    err = float(np.abs(got - want).max())
    rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
    assert np.isfinite(got).all() and err <= 2e-2 and rel <= 5e-3, (err, rel)


def test_forward_and_streaming_pass_the_checks(dev):
    w = C.Workload("dbg", B=1, H=2, D=128, T=7, frame_h=10, frame_w=20, Tc=3, To=1, P=2, F=128,
                   G=8, dtype="bf16", seed=23)
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    L = w.frame_tokens
    out = rb.forward(q, k, v, Wq, bq, Wk, bk, P=w.P, frame_tokens=L, Tc=w.Tc, To=w.To)
    rb.sync_status(dev)  # raises on a failed check
    from hybrid_softmax_linear_chunked_b200.streaming import ChunkStream
    sess = ChunkStream(Wq, bq, Wk, bk, B=w.B, P=w.P, frame_tokens=L, Tc=w.Tc, To=w.To)
    outs = [sess.step(*(x[:, :, s * L:e * L].contiguous() for x in (q, k, v))).clone()
            for (_, s, e) in w.chunk_bounds()]
    rb.sync_status(dev)
    stream_out = torch.cat(outs, dim=2)
    for h in range(w.H):
        pq = O.feature_map(f64(inp.q[0, h]), f64(inp.Wq[h]), f64(inp.bq[h]), w.P)
        pk = O.feature_map(f64(inp.k[0, h]), f64(inp.Wk[h]), f64(inp.bk[h]), w.P)
        want = O.hybrid_attention_quadratic(f64(inp.q[0, h]), f64(inp.k[0, h]),
                                            f64(inp.v[0, h]), pq, pk, L, w.Tc, w.To)
        check(f64(out[0, h]), want)
        check(f64(stream_out[0, h]), want)


def test_backward_passes_the_checks(dev):
    w = C.Workload("dbg bwd", B=1, H=2, D=128, T=7, frame_h=8, frame_w=10, Tc=3, To=1, P=2,
                   F=128, G=8, dtype="bf16", seed=29)
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    kw = dict(P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To)
    dout = torch.randn(inp.q.shape, generator=torch.Generator().manual_seed(3)).to(
        torch.bfloat16).to(dev)

    def grads():
        out, lse = rb.forward_train(*t, **kw)
        g = rb.backward(*t, out, lse, dout, **kw)
        rb.sync_status(dev)  # raises on a failed check
        return {n: g[n].detach().clone() for n in ("dq", "dk", "dv", "dWq", "dWk")}

    checked = grads()
    rb.use_library(build.build())
    try:
        plain = grads()
    finally:
        rb.use_library(build.build(debug_bounds=True))
    for n, x in checked.items():
        y = plain[n]
        # same kernels and arithmetic; the split-K GEMMs add in a varying order
        assert torch.isfinite(x).all(), n
        assert float((x - y).norm() / y.norm()) <= 1e-5, n


def test_out_of_range_store_is_caught(dev):
    n, bad = 1000, 1008
    buf = torch.zeros(n + 64, dtype=torch.float32, device=dev)
    rb.selftest_bounds(buf, n, bad)
    with pytest.raises(rb.RehyatError) as e:
        rb.sync_status(dev)
    assert e.value.status == -8 and "value 1008" in str(e.value)
    host = buf.cpu()
    assert bool((host[:n] == 1).all()) and float(host[bad]) == 0.0  # the store was skipped
    rb.sync_status(dev)  # the word was cleared
