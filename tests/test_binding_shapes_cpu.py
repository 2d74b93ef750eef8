"""The binding refuses tensors whose shapes disagree with what the library will read (the C ABI
takes sizes from the other arguments), before anything is enqueued.  On a CPU-only machine a call
with consistent shapes gets as far as the device check, so each entry is checked both ways:
consistent CPU tensors fail at the device check, an inconsistent one fails at the shape check."""
import pytest
import torch

from hybrid_softmax_linear_chunked_b200 import binding as rb

B, H, D, F, G, L, T, Tc, To = 1, 2, 128, 128, 8, 16, 6, 3, 1
N = T * L
DEVICE = "CUDA device"
SHAPE = "shape|rows|frames"


@pytest.fixture(scope="module", autouse=True)
def lib():
    return rb.load()


def x(rows, d=D, dtype=torch.bfloat16):
    return torch.zeros(B, H, rows, d, dtype=dtype)


def weights():
    return (torch.zeros(H, G, F // G, D // G), torch.zeros(H, F),
            torch.zeros(H, G, F // G, D // G), torch.zeros(H, F))


def test_forward_shapes():
    Wq, bq, Wk, bk = weights()
    kw = dict(P=2, frame_tokens=L, Tc=Tc, To=To)
    with pytest.raises(ValueError, match=DEVICE):
        rb.forward(x(N), x(N), x(N), Wq, bq, Wk, bk, **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.forward(x(N), x(N - L), x(N), Wq, bq, Wk, bk, **kw)        # k shorter than q
    with pytest.raises(ValueError, match=SHAPE):
        rb.forward(x(N), x(N), x(N), Wq, bq, Wk, bk, out=x(N - 1), **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.forward(x(N), x(N), x(N), Wq, torch.zeros(H, F - 1), Wk, bk, **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.forward(x(N), x(N), x(N), Wq, bq, torch.zeros(H, G, F // G, 8), bk, **kw)
    with pytest.raises(ValueError, match="weights"):
        rb.forward(x(N), x(N), x(N), torch.zeros(H, G, F // G, 8), bq, Wk, bk, **kw)


def test_phase_shapes():
    Wq, bq, Wk, bk = weights()
    kw = dict(P=2, frame_tokens=L, Tc=Tc, To=To)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match=DEVICE):
        rb.forward_states(x(N), x(N), Wk, bk, workspace=ws, **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.forward_states(x(N), x(N + L), Wk, bk, workspace=ws, **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.forward_states(x(N + 3), x(N + 3), Wk, bk, workspace=ws, **kw)   # not whole frames
    with pytest.raises(ValueError, match=DEVICE):
        rb.forward_phiq(x(N), Wq, bq, workspace=ws, **kw)
    d = rb.Dims(B, H, D, F, G, 2, 0)
    with pytest.raises(ValueError, match=DEVICE):
        rb.forward_attend(x(N), x(N), x(N), dims=d, frame_tokens=L, Tc=Tc, To=To, workspace=ws,
                          out=x(N))
    with pytest.raises(ValueError, match=SHAPE):
        rb.forward_attend(x(N), x(N), x(N - L), dims=d, frame_tokens=L, Tc=Tc, To=To,
                          workspace=ws, out=x(N))


def test_streaming_step_shapes():
    Wq, bq, Wk, bk = weights()
    S, Z = torch.zeros(B, H, F, D), torch.zeros(B, H, F)
    kw = dict(P=2, frame_tokens=L, To=To)
    q = x(Tc * L)
    win = x((To + Tc) * L)           # second chunk: one overlap frame plus its three frames
    for fn in (rb.chunk_forward, rb.chunk_forward_static):
        with pytest.raises(ValueError, match=DEVICE):
            fn(q, win, win, Wq, bq, Wk, bk, S, Z, frames_before=Tc, **kw)
        with pytest.raises(ValueError, match=DEVICE):     # first chunk: no overlap frames
            fn(q, q, q, Wq, bq, Wk, bk, S, Z, frames_before=0, **kw)
        with pytest.raises(ValueError, match=SHAPE):      # window without its overlap frame
            fn(q, q, q, Wq, bq, Wk, bk, S, Z, frames_before=Tc, **kw)
        with pytest.raises(ValueError, match=SHAPE):
            fn(q, win, win, Wq, bq, Wk, bk, S, torch.zeros(B, H, F + 1), frames_before=Tc, **kw)
    carry = x(To * L)
    with pytest.raises(ValueError, match=DEVICE):
        rb.chunk_forward_carry(q, q, q, Wq, bq, Wk, bk, S, Z, carry, carry, frames_before=Tc,
                               **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.chunk_forward_carry(q, q, q, Wq, bq, Wk, bk, S, Z, carry, x(2 * L), frames_before=Tc,
                               **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.chunk_forward_carry(q, win, win, Wq, bq, Wk, bk, S, Z, carry, carry,
                               frames_before=Tc, **kw)


def test_training_shapes():
    Wq, bq, Wk, bk = weights()
    kw = dict(P=2, frame_tokens=L, Tc=Tc, To=To)
    lse = torch.zeros(B, H, N)
    with pytest.raises(ValueError, match=DEVICE):
        rb.forward_train(x(N), x(N), x(N), Wq, bq, Wk, bk, **kw)
    with pytest.raises(ValueError, match=DEVICE):
        rb.backward(x(N), x(N), x(N), Wq, bq, Wk, bk, x(N), lse, x(N), **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.backward(x(N), x(N), x(N), Wq, bq, Wk, bk, x(N), torch.zeros(B, H, N - 1), x(N), **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.backward(x(N), x(N), x(N), Wq, bq, Wk, bk, x(N), lse, x(N - L), **kw)


def test_segment_shapes():
    Wq, bq, Wk, bk = weights()
    kw = dict(T=T, P=2, frame_tokens=L, Tc=Tc, To=To)
    ws = torch.zeros(16, dtype=torch.uint8)
    # chunks [1, 2): queries frames [3, 6), keys [2, 6)
    with pytest.raises(ValueError, match=DEVICE):
        rb.segment_states(x(4 * L), x(4 * L), Wk, bk, c0=1, c1=2, workspace=ws, **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.segment_states(x(3 * L), x(3 * L), Wk, bk, c0=1, c1=2, workspace=ws, **kw)
    S_pre, Z_pre = torch.zeros(1, B, H, F, D), torch.zeros(1, B, H, F)
    with pytest.raises(ValueError, match=DEVICE):
        rb.segment_attend(x(3 * L), x(4 * L), x(4 * L), Wq, bq, c0=1, c1=2, workspace=ws,
                          S_prefix=S_pre, Z_prefix=Z_pre, **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.segment_attend(x(4 * L), x(4 * L), x(4 * L), Wq, bq, c0=1, c1=2, workspace=ws, **kw)
    with pytest.raises(ValueError, match=SHAPE):
        rb.segment_attend(x(3 * L), x(4 * L), x(4 * L), Wq, bq, c0=1, c1=2, workspace=ws,
                          S_prefix=torch.zeros(1, B, H, F, D - 1), Z_prefix=Z_pre, **kw)
