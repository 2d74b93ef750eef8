"""Pins of the float64 backward oracle against things other than itself:
* central finite differences of the forward oracle (every input, both feature maps);
* torch autograd through scaled_dot_product_attention (float64) for a single chunk;
* torch autograd through a torch restatement of normalised linear attention with conv1d +
  softplus-power (or elu + 1) feature maps when the softmax window is empty.
A mutation test plants plausible mistakes in a copy of the backward oracle."""
import math
import types

import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O
import oracle.rehyat_oracle_backward as OB


def _problem(rng, T, L, D, F, G, bias=0.1):
    n = T * L
    q, k, v = (rng.standard_normal((n, D)) for _ in range(3))
    Wq = rng.standard_normal((G, F // G, D // G)) * math.sqrt(G / D)
    Wk = rng.standard_normal((G, F // G, D // G)) * math.sqrt(G / D)
    bq = np.full(F, bias) + 0.05 * rng.standard_normal(F)
    bk = np.full(F, bias) + 0.05 * rng.standard_normal(F)
    dout = rng.standard_normal((n, D))
    return [q, k, v, Wq, bq, Wk, bk], dout


def _loss(args, dout, P, L, Tc, To, kind):
    q, k, v, Wq, bq, Wk, bk = args
    pq, pk = O.feature_map(q, Wq, bq, P, kind), O.feature_map(k, Wk, bk, P, kind)
    return float(np.sum(dout * O.hybrid_attention_quadratic(q, k, v, pq, pk, L, Tc, To)))


def check_finite_differences(mod):
    rng = np.random.default_rng(21)
    for (T, L, Tc, To, P, kind) in [(4, 3, 2, 1, 2, O.PHI_POLY), (5, 2, 2, 2, 3, O.PHI_POLY),
                                    (4, 3, 2, 1, 1, O.PHI_ELU1)]:
        args, dout = _problem(rng, T, L, 8, 8, 2)
        grads = mod.hybrid_attention_backward(*args, P, L, Tc, To, dout, kind)
        for a, g in zip(args, grads):
            d = rng.standard_normal(a.shape)
            h = 1e-5
            plus = [x + h * d if x is a else x for x in args]
            minus = [x - h * d if x is a else x for x in args]
            fd = (_loss(plus, dout, P, L, Tc, To, kind) - _loss(minus, dout, P, L, Tc, To, kind)) / (2 * h)
            an = float(np.sum(g * d))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (T, L, Tc, To, P, kind, fd, an)


def check_single_chunk_sdpa(mod):
    rng = np.random.default_rng(22)
    T, L = 3, 4
    args, dout = _problem(rng, T, L, 16, 16, 4)
    grads = mod.hybrid_attention_backward(*args, 2, L, T, 0, dout)
    q, k, v = (torch.tensor(x, requires_grad=True) for x in args[:3])
    o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0]
    (o * torch.from_numpy(dout)).sum().backward()
    for g, t in zip(grads[:3], (q, k, v)):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-10, atol=1e-12)
    for g in grads[3:]:
        assert np.abs(g).max() == 0.0  # no linear region: phi gets no gradient


def _torch_phi(x, W, b, P, kind):
    G, Fg, Dg = W.shape
    u = torch.nn.functional.conv1d(x.T[None], W.reshape(G * Fg, Dg, 1), bias=b, groups=G)[0].T
    if kind == O.PHI_ELU1:
        return torch.nn.functional.elu(u) + 1.0
    parts = torch.tensor_split(u, P, dim=1)
    return torch.cat([torch.nn.functional.softplus(p_) ** (i + 1) for i, p_ in enumerate(parts)], dim=1)


def check_linear_only_autograd(mod):
    rng = np.random.default_rng(23)
    T, L = 3, 3
    for kind, P in [(O.PHI_POLY, 2), (O.PHI_POLY, 3), (O.PHI_ELU1, 1)]:
        args, dout = _problem(rng, T, L, 8, 8, 2)
        M = np.full((T, T), O.SET_LINEAR, dtype=np.int8)
        pq = O.feature_map(args[0], args[3], args[4], P, kind)
        pk = O.feature_map(args[1], args[5], args[6], P, kind)
        _, _, dv, dpq, dpk = mod.hybrid_attention_masked_backward(args[0], args[1], args[2], pq, pk,
                                                                  L, M, dout)
        dxq, dWq, dbq = mod.feature_map_backward(args[0], args[3], args[4], P, dpq, kind)
        dxk, dWk, dbk = mod.feature_map_backward(args[1], args[5], args[6], P, dpk, kind)
        ts = [torch.tensor(x, requires_grad=True) for x in args]
        q, k, v, Wq, bq, Wk, bk = ts
        fq, fk = _torch_phi(q, Wq, bq, P, kind), _torch_phi(k, Wk, bk, P, kind)
        o = (fq @ (fk.T @ v)) / (fq @ fk.sum(0))[:, None]
        (o * torch.from_numpy(dout)).sum().backward()
        for g, t in zip((dxq, dxk, dv, dWq, dbq, dWk, dbk), (q, k, v, Wq, bq, Wk, bk)):
            np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-10, atol=1e-12)


PINS = [check_finite_differences, check_single_chunk_sdpa, check_linear_only_autograd]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_backward_pin(pin):
    pin(OB)


MUTATIONS = [
    ("output term dropped from dL/dw",
     "g = (dout[rows] @ v.T - np.sum(dout[rows] * o, axis=1, keepdims=True)) / den",
     "g = (dout[rows] @ v.T) / den"),
    ("1/sqrt(D) missing in dq", "dq[rows] += ds @ k[sm] / math.sqrt(D)", "dq[rows] += ds @ k[sm]"),
    ("dv not normalised", "dv += (weights / den).T @ dout[rows]", "dv += weights.T @ dout[rows]"),
    ("linear gradient without the shift", "gl = g[:, li] * shift", "gl = g[:, li]"),
    ("softplus derivative without the sigmoid",
     "p * softplus(us) ** (p - 1) * sig[:, start:start + size]", "p * softplus(us) ** (p - 1)"),
    ("elu + 1 derivative taken as 1", "np.where(u > 0, 1.0, np.exp(np.minimum(u, 0.0)))",
     "np.ones_like(u)"),
    ("weight gradient transposed", "dW[g] = dug.T @ x[:, g * Dg:(g + 1) * Dg]",
     "dW[g] = (x[:, g * Dg:(g + 1) * Dg].T @ dug)[:Fg, :Dg] if Fg == Dg else dug.T @ x[:, g * Dg:(g + 1) * Dg] * 2"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_backward_mistake_is_caught(desc, old, new):
    src = open(OB.__file__).read()
    assert src.count(old) == 1, f"mutation anchor not unique for: {desc}"
    mod = types.ModuleType("oracle.mutant_backward")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), "mutant_backward", "exec"), mod.__dict__)
    failed = []
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught: {desc}"
