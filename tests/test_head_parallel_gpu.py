"""Head/batch sharding on one GPU: the ranks' shares of the B*H (batch, head) units run one after
another through HeadSharded (no kernel waits on another), and the assembled output must be
bit-identical to the one-call forward over all units.  The fold's token splits depend only on
the sequence shape, so a unit is computed the same way whichever units share its call."""
import pytest
import torch

from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.head_parallel import HeadSharded
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


SMALL = C.Workload("heads small", B=2, H=3, D=128, T=7, frame_h=10, frame_w=20, Tc=3, To=1, P=2,
                   F=128, G=8, dtype="bf16", seed=17)


@pytest.mark.parametrize("w,worlds", [(SMALL, (2, 4, 6)), (C.WAN_480P_5S, (2, 3, 8))],
                         ids=["B2_H3_200tok", "480p5s"])
def test_head_shards_bit_exact(dev, w, worlds):
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    kw = dict(P=w.P, frame_tokens=w.frame_tokens, Tc=w.Tc, To=w.To)
    full = rb.forward(q, k, v, Wq, bq, Wk, bk, **kw)
    rb.sync_status(dev)
    for world in worlds:
        got = torch.full_like(q, float("nan"))
        got_units = got.view(1, w.B * w.H, *q.shape[2:])
        for r in range(world):
            hs = HeadSharded(Wq, bq, Wk, bk, B=w.B, H=w.H, rank=r, world=world, **kw)
            out_s = hs.forward(hs.shard(q), hs.shard(k), hs.shard(v))
            got_units[:, hs.u0:hs.u1] = out_s
        rb.sync_status(dev)
        assert torch.equal(got, full), f"{world} shards differ from the one-call forward"
