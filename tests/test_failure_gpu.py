"""Failure detection on the GPU without a fault: a kernel's bounded wait runs out on a barrier
that nothing arrives on, the host reads REHYAT_ERR_TIMEOUT from the device error word, and the
context stays usable for the next forward."""
import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_softmax_linear_chunked_b200 import build
    build.build()
    rb.load()
    return torch.device("cuda", 0)


def test_wait_timeout_is_reported_and_cleared(dev):
    rb.sync_status(dev)                     # nothing pending
    rb.selftest_wait_timeout(20_000_000, dev)
    with pytest.raises(rb.RehyatError) as e:
        rb.sync_status(dev)
    assert e.value.status == -6, str(e.value)
    rb.sync_status(dev)                     # the error word was cleared

    # the context still runs the hybrid attention correctly
    w = C.Workload("after-timeout", B=1, H=1, D=128, T=4, frame_h=8, frame_w=10, Tc=2, To=1,
                   P=2, F=128, G=8, dtype="bf16", seed=21)
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    out = torch.full_like(q, float("nan"))
    rb.forward(q, k, v, Wq, bq, Wk, bk, P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To,
               out=out)
    rb.sync_status(dev)
    f = lambda t: t.detach().to("cpu", torch.float64).numpy()  # noqa: E731
    qh, kh, vh = f(inp.q[0, 0]), f(inp.k[0, 0]), f(inp.v[0, 0])
    want = O.hybrid_attention_quadratic(qh, kh, vh, O.feature_map(qh, f(inp.Wq[0]), f(inp.bq[0]), w.P),
                                        O.feature_map(kh, f(inp.Wk[0]), f(inp.bk[0]), w.P),
                                        w.frame_tokens, w.Tc, w.To)
    got = f(out[0, 0])
    assert np.isfinite(got).all()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 5e-3
