"""Float64 CPU oracle for the backward pass of ReHyAt hybrid attention.

TEST INFRASTRUCTURE ONLY, like rehyat_oracle.py: only the tests, the smoke check and the
CPU-baseline leg of the benchmark may import it; it imports nothing from the CUDA path.

The pages give the forward only ("ReHyAt overview" §2.2.1: output = (softmax part + linear part)
/ (softmax normaliser + linear normaliser); §2.2.2 the feature map; §3.1.1 trains phi_q and
phi_k by distillation and §3.1.2 fine-tunes the model, which both need these gradients).  This module is the
derivative of that definition, taken term by term on the explicit weights of the quadratic form
(every key materialised), so that a reader can check it against the forward by eye:

    w_ij  = e^{s_ij - mu_i}                      (j in T_S(i)),  s_ij = q_i . k_j / sqrt(D)
    w_ij  = (phi_q_i . phi_k_j) e^{-mu_i}         (j in T_L(i))
    o_i   = sum_j w_ij v_j / den_i,   den_i = sum_j w_ij

For a loss with gradient dO_i = dL/do_i:

    dL/dw_ij = (dO_i . v_j - dO_i . o_i) / den_i                 =: g_ij
    dv_j     = sum_i (w_ij / den_i) dO_i
    ds_ij    = g_ij w_ij                 (softmax pairs; mu_i cancels in the ratio)
    dq_i    += sum_j ds_ij k_j / sqrt(D),  dk_j += sum_i ds_ij q_i / sqrt(D)
    dphi_q_i = sum_j g_ij e^{-mu_i} phi_k_j,  dphi_k_j = sum_i g_ij e^{-mu_i} phi_q_i  (linear pairs)

and through the feature map phi = f(u), u_g = x_g W[g]^T + b:

    du = dphi * f'(u);  dx_g = du_g W[g];  dW[g] = du_g^T x_g;  db = sum over tokens of du
    f'(u) = p softplus(u)^(p-1) sigmoid(u) on part p (polynomial map);  1 (u > 0) or e^u (elu+1).
"""
from __future__ import annotations

import math

import numpy as np

from .rehyat_oracle import (PHI_ELU1, PHI_POLY, SET_LINEAR, SET_SOFTMAX, feature_map,
                            part_sizes, rehyat_mask, softplus)

__all__ = ["hybrid_attention_masked_backward", "feature_map_backward",
           "hybrid_attention_backward"]


def hybrid_attention_masked_backward(q, k, v, phi_q, phi_k, frame_tokens: int, M, dout):
    """Gradients of sum(dout * o) for the masked quadratic form (any frame-level set
    assignment M).  Returns (dq, dk, dv, dphi_q, dphi_k); dq and dk hold the softmax-logit
    paths only (the feature-map paths come back through dphi_q, dphi_k)."""
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    phi_q = np.asarray(phi_q, np.float64); phi_k = np.asarray(phi_k, np.float64)
    dout = np.asarray(dout, np.float64)
    n, D = q.shape
    L = frame_tokens
    T = n // L
    key_frame = np.arange(n) // L
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    dphi_q = np.zeros_like(phi_q); dphi_k = np.zeros_like(phi_k)
    for tq in range(T):
        rows = slice(tq * L, (tq + 1) * L)
        sm = M[tq][key_frame] == SET_SOFTMAX
        li = M[tq][key_frame] == SET_LINEAR
        if not (sm.any() or li.any()):
            continue
        weights = np.zeros((L, n))
        if sm.any():
            logits = q[rows] @ k[sm].T / math.sqrt(D)
            mu = logits.max(axis=1, keepdims=True)
            weights[:, sm] = np.exp(logits - mu)
        else:
            mu = np.zeros((L, 1))
        shift = np.exp(-mu)
        if li.any():
            weights[:, li] = (phi_q[rows] @ phi_k[li].T) * shift
        den = weights.sum(axis=1, keepdims=True)
        o = (weights @ v) / den
        g = (dout[rows] @ v.T - np.sum(dout[rows] * o, axis=1, keepdims=True)) / den
        dv += (weights / den).T @ dout[rows]
        if sm.any():
            ds = g[:, sm] * weights[:, sm]
            dq[rows] += ds @ k[sm] / math.sqrt(D)
            dk[sm] += ds.T @ q[rows] / math.sqrt(D)
        if li.any():
            gl = g[:, li] * shift
            dphi_q[rows] += gl @ phi_k[li]
            dphi_k[li] += gl.T @ phi_q[rows]
    return dq, dk, dv, dphi_q, dphi_k


def feature_map_backward(x, W, bias, P: int, dphi, kind: str = PHI_POLY):
    """Gradients (dx, dW, db) of sum(dphi * phi(x)) for the feature map of rehyat_oracle."""
    x = np.asarray(x, np.float64); W = np.asarray(W, np.float64)
    dphi = np.asarray(dphi, np.float64)
    n, D = x.shape
    G, Fg, Dg = W.shape
    F = G * Fg
    u = np.empty((n, F))
    for g in range(G):
        u[:, g * Fg:(g + 1) * Fg] = x[:, g * Dg:(g + 1) * Dg] @ W[g].T
    if bias is not None:
        u = u + np.asarray(bias, np.float64)[None, :]
    if kind == PHI_ELU1:
        fprime = np.where(u > 0, 1.0, np.exp(np.minimum(u, 0.0)))
    else:
        fprime = np.empty_like(u)
        sig = 0.5 * (1.0 + np.tanh(0.5 * u))  # logistic sigmoid, overflow-free
        start = 0
        for p, size in enumerate(part_sizes(F, P), start=1):
            us = u[:, start:start + size]
            fprime[:, start:start + size] = p * softplus(us) ** (p - 1) * sig[:, start:start + size]
            start += size
    du = dphi * fprime
    dx = np.zeros_like(x)
    dW = np.zeros_like(W)
    for g in range(G):
        dug = du[:, g * Fg:(g + 1) * Fg]
        dx[:, g * Dg:(g + 1) * Dg] = dug @ W[g]
        dW[g] = dug.T @ x[:, g * Dg:(g + 1) * Dg]
    db = du.sum(axis=0)
    return dx, dW, db


def hybrid_attention_backward(q, k, v, Wq, bq, Wk, bk, P: int, frame_tokens: int, Tc: int,
                              To: int, dout, kind: str = PHI_POLY):
    """All gradients of sum(dout * out) for one (b, h) of the standard chunk schedule:
    (dq, dk, dv, dWq, dbq, dWk, dbk)."""
    phi_q = feature_map(q, Wq, bq, P, kind)
    phi_k = feature_map(k, Wk, bk, P, kind)
    T = np.asarray(q).shape[0] // frame_tokens
    M = rehyat_mask(T, Tc, To)
    dq, dk, dv, dpq, dpk = hybrid_attention_masked_backward(q, k, v, phi_q, phi_k, frame_tokens,
                                                            M, dout)
    dxq, dWq, dbq = feature_map_backward(q, Wq, bq, P, dpq, kind)
    dxk, dWk, dbk = feature_map_backward(k, Wk, bk, P, dpk, kind)
    return dq + dxq, dk + dxk, dv, dWq, dbq, dWk, dbk
