"""The backward pass (and the forward's row statistics it needs) on the GPU against the float64
oracle of the gradients, on seeded inputs.

Tolerances, from the rounding the GPU path does.  Every tensor-core operand that is not an input
is rounded to bf16 (relative error at most 2^-9 per element); products accumulate in fp32, whose
rounding (2^-24 per add) is negligible next to it.  A gradient element is a sum of terms, and the
rounding errors of different terms are independent, so its relative error is at most the
per-term bound times the sum's cancellation ratio R = (norm of the terms) / (norm of their sum).
* dq, dk, dv: a term passes through at most two bf16 roundings (P or dS as a GEMM operand, and
  the bf16 output o inside D = dO . o), 2 * 2^-9 = 3.9e-3; REL_L2 = 1e-2 allows R up to 2.5.
* dW, db: sums over every token of du x^T, du passing through three roundings (phi, the
  dS / P upstream, du itself as the GEMM operand), 3 * 2^-9 = 5.9e-3; terms of both signs cancel
  across tokens, and REL_L2_W = 2.5e-2 allows R up to 4.3.
* lse (log2 units): the denominators are fp32 sums of fp32 exponentials plus phi_q . Z with
  bf16 phi_q, within 2^-9 relative, i.e. 2.8e-3 in log2 units; bound 1e-2.
Measured: dq, dk, dv 1.3e-3 to 2.1e-3; dW, db 2.5e-3 to 8.6e-3; lse within 2.5e-3."""
import math

import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
import oracle.rehyat_oracle_backward as OB
from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import configs as C
from hybrid_softmax_linear_chunked_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu
REL_L2 = 1e-2
REL_L2_W = 2.5e-2


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
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


CASES = [
    # T, fh, fw, Tc, To, P, G, B, H, bias, phi
    (7, 30, 52, 3, 1, 2, 8, 1, 2, 0.0, "poly"),   # 1560-token frames of the 480x832 workload
    (7, 30, 52, 3, 1, 2, 8, 1, 1, -30.0, "poly"),  # ... with the linear branch switched off
    (7, 8, 10, 3, 1, 2, 8, 1, 2, 0.1, "poly"),
    (8, 6, 12, 3, 1, 3, 8, 2, 1, 0.0, "poly"),    # ragged last chunk, B = 2
    (6, 8, 8, 2, 2, 2, 16, 1, 2, 0.2, "poly"),
    (5, 8, 10, 1, 0, 1, 4, 1, 1, 0.1, "poly"),    # Tc = 1, no overlap
    (7, 8, 10, 3, 1, 1, 8, 1, 2, 0.1, "elu1"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"T{c[0]}_L{c[1]*c[2]}_Tc{c[3]}_To{c[4]}_P{c[5]}_G{c[6]}_B{c[7]}_{c[10]}" for c in CASES])
def test_backward_matches_oracle(dev, case):
    T, fh, fw, Tc, To, P, G, B, H, bias, phi = case
    w = C.Workload("bwd", B=B, H=H, D=128, T=T, frame_h=fh, frame_w=fw, Tc=Tc, To=To, P=P,
                   F=128, G=G, dtype="bf16", bias=bias, seed=41 + T, phi=phi)
    inp = make_inputs(w)
    t = [x.to(dev) for x in (inp.q, inp.k, inp.v, inp.Wq, inp.bq, inp.Wk, inp.bk)]
    kw = dict(P=P, phi=w.phi_code, frame_tokens=w.frame_tokens, Tc=Tc, To=To)
    out, lse = rb.forward_train(*t, **kw)
    dout = torch.randn(out.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    g = rb.backward(*t, out, lse, dout.to(dev), **kw)
    rb.sync_status(dev)
    kind = O.PHI_ELU1 if phi == "elu1" else O.PHI_POLY
    L = w.frame_tokens
    acc = {n: 0.0 for n in ("dWq", "dbq", "dWk", "dbk")}
    errs = {}
    for h in range(H):
        sums = None
        for b in range(B):
            args = [f64(inp.q[b, h]), f64(inp.k[b, h]), f64(inp.v[b, h]), f64(inp.Wq[h]),
                    f64(inp.bq[h]), f64(inp.Wk[h]), f64(inp.bk[h])]
            want = OB.hybrid_attention_backward(*args, P, L, Tc, To, f64(dout[b, h]), kind)
            for name, wv in zip(("dq", "dk", "dv"), want[:3]):
                errs[f"{name} b{b} h{h}"] = rel_l2(f64(g[name][b, h]), wv)
            sums = list(want[3:]) if sums is None else [s + x for s, x in zip(sums, want[3:])]
            # the forward's row statistic: log2 of sum_window e^s + phi_q . Z
            pq = O.feature_map(args[0], args[3], args[4], P, kind)
            pk = O.feature_map(args[1], args[5], args[6], P, kind)
            lse_want = np.empty(w.N)
            for (wf, s, e) in w.chunk_bounds():
                lg = args[0][s * L:e * L] @ args[1][wf * L:e * L].T / math.sqrt(128)
                den = np.exp(lg).sum(axis=1) + pq[s * L:e * L] @ pk[:wf * L].sum(axis=0)
                lse_want[s * L:e * L] = np.log2(den)
            errs[f"lse b{b} h{h} (abs)"] = float(np.abs(f64(lse[b, h]) - lse_want).max())
        # with bias -30 the feature maps are ~e^(u - 30): their gradients are checked where the
        # linear branch carries weight, not here
        if bias > -10:
            for name, wv in zip(("dWq", "dbq", "dWk", "dbk"), sums):
                errs[f"{name} h{h}"] = rel_l2(f64(g[name][h]), wv)
    msg = " ".join(f"{k}={v:.2e}" for k, v in errs.items())
    print(msg)
    for k, v in errs.items():
        assert np.isfinite(v), msg
        if "lse" in k:
            assert v <= 1e-2, msg
        elif k.startswith(("dW", "db")):
            assert v <= REL_L2_W, msg
        else:
            assert v <= REL_L2, msg
