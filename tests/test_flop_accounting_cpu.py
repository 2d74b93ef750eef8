"""The algorithmic work the bench divides by its times (the roofline's numerator), counted a second
way: per query frame and key frame, from the method's definition ("ReHyAt overview" §2.2.1: a
query takes softmax over the keys of its chunk and the To frames before it, and reads the
linear state of every earlier key; §2.3: the state is the sum of phi_k(k) v^T over the folded
keys), against the per-chunk sums of `configs.Workload`.

Per (query token, key token) pair inside the window: 2D (q.k) + 2D (p v) FLOPs.  Per query whose
chunk has a linear region: 2FD + 2F (phi_q . S, phi_q . Z).  Per folded key: 2FD + F (phi_k v^T,
phi_k).  Per token whose feature map is consumed: 2 D F / G.  Exponentials count zero."""
import itertools

import pytest

from hybrid_softmax_linear_chunked_b200 import configs as C


def brute(w: C.Workload, streaming: bool):
    L, D, F, G, T, Tc, To = w.frame_tokens, w.D, w.F, w.G, w.T, w.Tc, w.To
    softmax = readout = 0
    q_lin = 0
    window_start = []
    for tq in range(T):
        c = tq // Tc
        lo, hi = max(0, c * Tc - To), min((c + 1) * Tc, T)
        window_start.append(lo)
        for tk in range(T):
            if lo <= tk < hi:
                softmax += 4 * D * L * L
        if lo > 0:
            readout += L * (2 * F * D + 2 * F)
            q_lin += L
    if streaming:
        # after every call the frames the next window (same overlap) no longer holds are folded;
        # after the last call that is every frame before its last To
        folded_frames = [tk for tk in range(T) if tk < max(0, T - To)]
    else:
        # the whole-sequence call folds the keys some chunk reads through its state
        folded_frames = [tk for tk in range(T) if any(tk < lo for lo in window_start)]
    folded = len(folded_frames) * L
    state = folded * (2 * F * D + F)
    phi = (q_lin + folded) * 2 * D * F // G
    tensor = softmax + q_lin * 2 * F * D
    return (softmax + readout + state + phi) * w.B * w.H, tensor * w.B * w.H


SHAPES = list(itertools.product([1, 2, 3, 5], [0, 1, 2], [1, 4, 7, 21]))


@pytest.mark.parametrize("Tc,To,T", SHAPES)
@pytest.mark.parametrize("streaming", [False, True])
def test_flops_match_pairwise_count(Tc, To, T, streaming):
    w = C.Workload("t", B=2, H=3, D=16, T=T, frame_h=2, frame_w=3, Tc=Tc, To=To, P=2, F=16, G=4,
                   dtype="bf16")
    total, tensor = brute(w, streaming)
    assert w.flops(streaming=streaming) == pytest.approx(total, rel=1e-12)
    assert w.attn_tensor_flops() == pytest.approx(tensor, rel=1e-12)


@pytest.mark.parametrize("w,flops,bytes_", [
    (C.TINY_F32, 8.97e5, 49e3),
    (C.WAN_480P_5S, 1.2354e12, 402.6e6),
    (C.WAN_480P_10S, 2.4301e12, 786e6),
    (C.WAN_720P_5S, 6.5058e12, 929e6),
    (C.WAN_480P_20S_STREAM, 9.8184e12, 3.105e9),
])
def test_workload_totals(w, flops, bytes_):
    # the totals as printed in the workload table (four or five significant digits)
    assert w.flops() == pytest.approx(flops, rel=6e-4)
    assert w.flops() == pytest.approx(brute(w, w.mode == "stream")[0], rel=1e-12)
    assert w.io_bytes() == pytest.approx(bytes_, rel=6e-3)


def test_attention_share_480p5s():
    # softmax 1.2111e12 + readout 1.11e10 on the tensor cores of the attention launch
    assert C.WAN_480P_5S.attn_tensor_flops() == pytest.approx(1.2111e12 + 1.11e10, rel=1e-3)
