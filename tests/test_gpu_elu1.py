"""The elu(u) + 1 feature map (the linear attention of the "ReHyAt overview" page, §2.1.2) on
every CUDA path, against the float64 oracle with the same map: the standalone feature map, the
whole-sequence forward (bf16 tensor-core path and fp32 path), the pages' own form (identity
grouped linear, elu + 1 of the raw token), and the streaming calls."""
import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs
from hybrid_softmax_linear_chunked_b200.streaming import ChunkStream

pytestmark = pytest.mark.gpu
ELU1 = rb.PHI_ELU1


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


def oracle_head(q, k, v, Wq, bq, Wk, bk, w):
    pq = O.feature_map(q, Wq, bq, w.P, O.PHI_ELU1)
    pk = O.feature_map(k, Wk, bk, w.P, O.PHI_ELU1)
    return O.hybrid_attention_quadratic(q, k, v, pq, pk, w.frame_tokens, w.Tc, w.To)


def forward(t, w, dev):
    q, k, v, Wq, bq, Wk, bk = t
    out = torch.full_like(q, float("nan"))
    rb.forward(q, k, v, Wq, bq, Wk, bk, P=w.P, phi=ELU1, frame_tokens=w.frame_tokens, Tc=w.Tc,
               To=w.To, out=out)
    rb.sync_status(dev)
    return out


@pytest.mark.parametrize("dtype,G", [("bf16", 8), ("bf16", 128), ("f32", 4)])
def test_featmap_elu1(dev, dtype, G):
    D = 128 if dtype == "bf16" else 32
    w = C.Workload("fm-elu1", B=1, H=2, D=D, T=1, frame_h=1, frame_w=200, Tc=1, To=0, P=1, F=D,
                   G=G, dtype=dtype, bias=0.2, seed=13, phi="elu1")
    inp = make_inputs(w)
    phi = rb.featmap(inp.q.to(dev), inp.Wq.to(dev), inp.bq.to(dev), 1, ELU1)
    for h in range(2):
        want = O.feature_map(f64(inp.q[0, h]), f64(inp.Wq[h]), f64(inp.bq[h]), 1, O.PHI_ELU1)
        tol = dict(rtol=8e-3, atol=1e-6) if dtype == "bf16" else dict(rtol=2e-6, atol=1e-7)
        np.testing.assert_allclose(f64(phi[0, h]), want, **tol)


@pytest.mark.parametrize("T,fh,fw,Tc,To", [(7, 10, 20, 3, 1), (5, 9, 15, 2, 2)])
def test_bf16_forward_elu1(dev, T, fh, fw, Tc, To):
    w = C.Workload("elu1", B=1, H=2, D=128, T=T, frame_h=fh, frame_w=fw, Tc=Tc, To=To, P=1,
                   F=128, G=8, dtype="bf16", bias=0.1, seed=14, phi="elu1")
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    out = forward(t, w, dev)
    for h in range(2):
        want = oracle_head(f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h]), f64(inp.Wq[h]),
                           f64(inp.bq[h]), f64(inp.Wk[h]), f64(inp.bk[h]), w)
        got = f64(out[0, h])
        assert np.isfinite(got).all()
        assert np.abs(got - want).max() <= 2e-2 and rel_l2(got, want) <= 5e-3


def test_bf16_elu1_of_raw_tokens(dev):
    """The pages' form: phi(x) = elu(x) + 1 of q and k themselves (G = D groups of 1 x 1
    weights equal to 1, no bias)."""
    w = C.Workload("elu1-raw", B=1, H=2, D=128, T=6, frame_h=8, frame_w=16, Tc=3, To=1, P=1,
                   F=128, G=128, dtype="bf16", seed=15, phi="elu1")
    inp = make_inputs(w)
    eye = torch.ones(2, 128, 1, 1)
    zero = torch.zeros(2, 128)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, eye, zero, eye, zero)]
    out = forward(t, w, dev)
    for h in range(2):
        q, k, v = f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h])
        eq = np.where(q > 0, q + 1, np.exp(q)); ek = np.where(k > 0, k + 1, np.exp(k))
        want = O.hybrid_attention_quadratic(q, k, v, eq, ek, w.frame_tokens, w.Tc, w.To)
        got = f64(out[0, h])
        assert np.abs(got - want).max() <= 2e-2 and rel_l2(got, want) <= 5e-3


def test_f32_forward_elu1(dev):
    w = C.Workload("elu1-f32", B=1, H=2, D=32, T=6, frame_h=4, frame_w=4, Tc=3, To=1, P=1, F=32,
                   G=4, dtype="f32", bias=0.1, seed=16, phi="elu1")
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    out = forward(t, w, dev)
    for h in range(2):
        want = oracle_head(f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h]), f64(inp.Wq[h]),
                           f64(inp.bq[h]), f64(inp.Wk[h]), f64(inp.bk[h]), w)
        assert rel_l2(f64(out[0, h]), want) <= 1e-5


def test_streaming_elu1(dev):
    w = C.Workload("elu1-stream", B=1, H=2, D=128, T=8, frame_h=6, frame_w=12, Tc=3, To=1, P=1,
                   F=128, G=8, dtype="bf16", bias=0.1, seed=17, phi="elu1")
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    sess = ChunkStream(Wq, bq, Wk, bk, B=1, P=1, phi=ELU1, frame_tokens=w.frame_tokens, Tc=w.Tc,
                       To=w.To)
    L = w.frame_tokens
    outs = [sess.step(q[:, :, s * L:e * L].contiguous(), k[:, :, s * L:e * L].contiguous(),
                      v[:, :, s * L:e * L].contiguous()).clone() for (_, s, e) in w.chunk_bounds()]
    rb.sync_status(dev)
    out = torch.cat(outs, dim=2)
    full = forward([q, k, v, Wq, bq, Wk, bk], w, dev)
    for h in range(2):
        want = oracle_head(f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h]), f64(inp.Wq[h]),
                           f64(inp.bq[h]), f64(inp.Wk[h]), f64(inp.bk[h]), w)
        assert rel_l2(f64(out[0, h]), want) <= 5e-3
    assert rel_l2(f64(out), f64(full)) <= 3e-3


def test_static_chunk_elu1(dev):
    """The workspace-free streaming entry computes phi_q inside the attention kernel."""
    w = C.Workload("elu1-static", B=1, H=2, D=128, T=6, frame_h=5, frame_w=10, Tc=3, To=1, P=1,
                   F=128, G=8, dtype="bf16", bias=0.1, seed=18, phi="elu1")
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    L = w.frame_tokens
    res = []
    for fn in (rb.chunk_forward, rb.chunk_forward_static):
        S = torch.zeros(1, 2, 128, 128, dtype=torch.float32, device=dev)
        Z = torch.zeros(1, 2, 128, dtype=torch.float32, device=dev)
        outs = []
        for (wf, s, e) in w.chunk_bounds():
            outs.append(fn(q[:, :, s * L:e * L].contiguous(), k[:, :, wf * L:e * L].contiguous(),
                           v[:, :, wf * L:e * L].contiguous(), Wq, bq, Wk, bk, S, Z, P=1,
                           phi=ELU1, frame_tokens=L, frames_before=s, To=w.To))
        rb.sync_status(dev)
        res.append(torch.cat(outs, dim=2))
    assert rel_l2(f64(res[1]), f64(res[0])) <= 3e-3
    for h in range(2):
        want = oracle_head(f64(inp.q[0, h]), f64(inp.k[0, h]), f64(inp.v[0, h]), f64(inp.Wq[h]),
                           f64(inp.bq[h]), f64(inp.Wk[h]), f64(inp.bk[h]), w)
        assert rel_l2(f64(res[1][0, h]), want) <= 5e-3
