"""rehyat_chunk_forward_static: the streaming step for callers that cannot allocate device
memory (a plugin whose host framework owns every allocation, or code that must not call
cudaMalloc while other work is being captured or replayed).  It takes no workspace and uses a
fixed scratch array inside the library instead.

Checked against the ordinary rehyat_chunk_forward (caller-provided workspace) on two calls in a
row, with the bf16 tolerances of the other parity tests.  The file name sorts last so that a run
that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3
STATE_REL = 1e-5


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_softmax_linear_chunked_b200 import build
    build.build()
    rb.load()
    return torch.device("cuda", 0)


def close_state(a, b, what):
    """S and Z are fp32 sums over thousands of tokens (Z reaches ~1e4): when the two calls split
    the fold differently the summation order differs, so they agree to fp32 rounding relative to
    their size, not to an absolute bound."""
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    err = np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert np.isfinite(a).all(), what + ": non-finite"
    assert err <= STATE_REL and rel <= STATE_REL, f"{what}: max-abs/max {err:.3e} rel-L2 {rel:.3e}"


def close(a, b, what):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    err = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert np.isfinite(a).all(), what + ": non-finite"
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {err:.3e} rel-L2 {rel:.3e}"


# (1, 74, 30, 52): the workspace call folds with two token splits, which do not fit the static
# scratch beside 74 heads' states and weights (17.05 MB), so the static call folds with one.
@pytest.mark.parametrize("B,H,fh,fw", [(1, 2, 10, 20), (2, 12, 30, 52), (1, 74, 30, 52)],
                         ids=["2heads_200tok", "24heads_1560tok", "74heads_1560tok_capped_splits"])
def test_static_scratch_matches_workspace_call(dev, B, H, fh, fw):
    w = C.Workload("no-alloc", B=B, H=H, D=128, T=6, frame_h=fh, frame_w=fw, Tc=3, To=1, P=2,
                   F=128, G=8, dtype="bf16", seed=21)
    inp = make_inputs(w)
    q, k, v, Wq, bq, Wk, bk = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk,
                                                   inp.bk))
    L = w.frame_tokens
    S_ref = torch.zeros(B, H, w.F, w.D, dtype=torch.float32, device=dev)
    Z_ref = torch.zeros(B, H, w.F, dtype=torch.float32, device=dev)
    S_st, Z_st = S_ref.clone(), Z_ref.clone()
    for (wf, s, e) in w.chunk_bounds():  # two calls in a row: frames 0-2, then frames 3-5
        qc = q[:, :, s * L:e * L].contiguous()
        kw = k[:, :, wf * L:e * L].contiguous()
        vw = v[:, :, wf * L:e * L].contiguous()
        kwargs = dict(P=w.P, frame_tokens=L, frames_before=s, To=w.To)
        ref = rb.chunk_forward(qc, kw, vw, Wq, bq, Wk, bk, S_ref, Z_ref, **kwargs)
        got = torch.full_like(qc, float("nan"))
        rb.chunk_forward_static(qc, kw, vw, Wq, bq, Wk, bk, S_st, Z_st, out=got, **kwargs)
        rb.sync_status(dev)
        close(got, ref, f"output of the chunk at frame {s}")
        close_state(S_st, S_ref, f"S after the chunk at frame {s}")
        close_state(Z_st, Z_ref, f"Z after the chunk at frame {s}")
