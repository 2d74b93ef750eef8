"""HostPipeline: batches from pinned host memory through the forward with the uploads, the
computation and the downloads on three streams.  Every step's output must equal the forward of
that step's own inputs (bit for bit: the kernels are deterministic), which fails if a buffer is
overwritten before its reader is done."""
import pytest
import torch

from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.host_pipeline import HostPipeline
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


@pytest.mark.parametrize("n", [1, 2, 5])
def test_pipeline_outputs_match_direct_forward(dev, n):
    w = C.Workload("pipe", B=1, H=2, D=128, T=7, frame_h=10, frame_w=20, Tc=3, To=1, P=2, F=128,
                   G=8, dtype="bf16", seed=3)
    kw = dict(P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To)
    batches = []
    for i in range(n):
        inp = make_inputs(w, seed=100 + i)
        batches.append([x.pin_memory() for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                 inp.bk)])
    outs = [torch.full(batches[0][0].shape, float("nan"), dtype=torch.bfloat16).pin_memory()
            for _ in range(n)]
    like_out = torch.empty(batches[0][0].shape, dtype=torch.bfloat16, device=dev)
    pipe = HostPipeline(lambda i, ins, o: rb.forward(*ins, out=o, **kw), batches[0], like_out,
                        dev)
    pipe.run(batches, outs)
    torch.cuda.current_stream(dev).synchronize()
    rb.sync_status(dev)
    for i in range(n):
        want = rb.forward(*(x.to(dev) for x in batches[i]), **kw).cpu()
        assert torch.equal(outs[i], want), f"step {i}"
