"""Pins of the float64 oracle against things other than itself.

What pins what:
* hand-derived worked examples (tests/golden/worked_examples.json) -> the output formula, the
  window/linear split, the overlap, the part powers, bidirectional softmax inside a chunk;
* torch conv1d(groups=G) + torch softplus                             -> the feature map;
* torch elu + 1 on the raw token (identity grouped linear)           -> the elu+1 feature map;
* the linear attention of the pages' §2.1.2 (phi = elu + 1, no chunks)
  and a scalar brute force with elu + 1                              -> the elu+1 hybrid;
* torch scaled_dot_product_attention (float64)                       -> the single-chunk case;
* normalised linear attention written with cumulative sums           -> the empty-window case;
* scalar brute force (own phi, own frame classification)             -> everything, tiny sizes;
* recurrent and streaming forms against the quadratic form           -> the fold;
* closed-form prefix sums                                            -> the states;
* invariants (convex combination, constant v, permutation within a frame).
A mutation test plants plausible mistakes in a copy of the oracle and checks that some pin fails.
"""
import json
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _val(s: str) -> float:
    env = {"sqrt2": math.sqrt(2.0), "ln4": math.log(4.0), "e": math.e, "ln": math.log}
    return float(eval(s.replace("^", "**"), {"__builtins__": {}}, env))


def _rand_problem(rng, T, L, D, F, G, bias=0.0, kscale=1.0):
    n = T * L
    q = rng.standard_normal((n, D))
    k = rng.standard_normal((n, D)) * kscale
    v = rng.standard_normal((n, D))
    Wq = rng.standard_normal((G, F // G, D // G)) * math.sqrt(G / D)
    Wk = rng.standard_normal((G, F // G, D // G)) * math.sqrt(G / D)
    bq = np.full(F, bias) + 0.1 * rng.standard_normal(F)
    bk = np.full(F, bias) + 0.1 * rng.standard_normal(F)
    return q, k, v, Wq, bq, Wk, bk


# ------------------------------------------------------------------------------------------
# pin checks, written against a module object so that the mutation test can reuse them
# ------------------------------------------------------------------------------------------

def check_golden(mod):
    g = json.load(open(GOLDEN))
    q = np.array([[_val(x) for x in r] for r in g["inputs"]["q"]])
    k = np.array([[_val(x) for x in r] for r in g["inputs"]["k"]])
    v = np.array([[_val(x) for x in r] for r in g["inputs"]["v"]])
    W = np.array([[[_val(x) for x in r] for r in blk] for blk in g["inputs"]["W"]])
    for case in g["cases"]:
        b = np.array([_val(x) for x in case["b"]])
        want = np.array([[_val(x) for x in r] for r in case["out"]])
        pq = mod.feature_map(q, W, b, case["P"])
        pk = mod.feature_map(k, W, b, case["P"])
        got = mod.hybrid_attention_quadratic(q, k, v, pq, pk, 1, case["Tc"], case["To"])
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13, err_msg=case["name"])
        got_r = mod.hybrid_attention_recurrent(q, k, v, pq, pk, 1, case["Tc"], case["To"])
        np.testing.assert_allclose(got_r, want, rtol=1e-13, atol=1e-13, err_msg=case["name"])
        got_b = mod.hybrid_attention_bruteforce(q, k, v, W, b, W, b, case["P"], 1, case["Tc"],
                                                case["To"])
        np.testing.assert_allclose(got_b, want, rtol=1e-13, atol=1e-13, err_msg=case["name"])


def check_featmap_conv1d(mod):
    rng = np.random.default_rng(1)
    for (D, F, G, P) in [(32, 32, 4, 2), (128, 128, 8, 3), (16, 24, 4, 1), (64, 32, 8, 2)]:
        x = rng.standard_normal((37, D))
        W = rng.standard_normal((G, F // G, D // G)) * math.sqrt(G / D) * 2
        b = rng.standard_normal(F)
        got = mod.feature_map(x, W, b, P)
        xt = torch.from_numpy(x).T[None]  # [1, D, n]
        u = torch.nn.functional.conv1d(xt, torch.from_numpy(W).reshape(F, D // G, 1),
                                       bias=torch.from_numpy(b), groups=G)[0].T
        parts = torch.tensor_split(u, P, dim=1)
        # torch softplus switches to the identity above threshold=20, where log1p(e^-x) < 2.1e-9
        want = torch.cat([torch.nn.functional.softplus(pp) ** (i + 1)
                          for i, pp in enumerate(parts)], dim=1).numpy()
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-8)


def check_single_chunk_is_softmax(mod):
    rng = np.random.default_rng(2)
    for (T, L, Tc, To) in [(4, 3, 4, 0), (3, 5, 7, 2), (1, 8, 1, 1)]:
        q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, 8, 8, 2)
        pq, pk = mod.feature_map(q, Wq, bq, 2), mod.feature_map(k, Wk, bk, 2)
        got = mod.hybrid_attention_quadratic(q, k, v, pq, pk, L, Tc, To)
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0]
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-12)
        got_r = mod.hybrid_attention_recurrent(q, k, v, pq, pk, L, Tc, To)
        np.testing.assert_allclose(got_r, want.numpy(), rtol=1e-12, atol=1e-12)


def check_linear_only(mod):
    """T_S empty: the hybrid reduces to normalised linear attention with the same phi."""
    rng = np.random.default_rng(3)
    T, L, D = 5, 3, 8
    q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, D, 8, 2)
    pq, pk = mod.feature_map(q, Wq, bq, 2), mod.feature_map(k, Wk, bk, 2)
    # every key visible, all linear
    M = np.full((T, T), mod.SET_LINEAR, dtype=np.int8)
    got = mod.hybrid_attention_masked(q, k, v, pq, pk, L, M)
    want = (pq @ (pk.T @ v)) / (pq @ pk.sum(axis=0))[:, None]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # causal by chunk (Tc = 2): query frame t sees key frames of chunks <= its own, all linear
    Tc = 2
    M = np.full((T, T), mod.SET_NONE, dtype=np.int8)
    for tq in range(T):
        M[tq, :min((tq // Tc + 1) * Tc, T)] = mod.SET_LINEAR
    got = mod.hybrid_attention_masked(q, k, v, pq, pk, L, M)
    kv = np.cumsum(np.einsum("nf,nd->nfd", pk, v), axis=0)
    ks = np.cumsum(pk, axis=0)
    want = np.empty_like(got)
    for i in range(T * L):
        last = min(((i // L) // Tc + 1) * Tc, T) * L - 1
        want[i] = (pq[i] @ kv[last]) / (pq[i] @ ks[last])
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def check_bruteforce(mod):
    rng = np.random.default_rng(4)
    cases = [(6, 16, 32, 32, 4, 3, 1, 2)]  # the tiny workload's shape
    for _ in range(10):
        cases.append((int(rng.integers(1, 8)), int(rng.integers(1, 6)), 4, 4, 2,
                      int(rng.integers(1, 5)), int(rng.integers(0, 4)), int(rng.integers(1, 4))))
    for (T, L, D, F, G, Tc, To, P) in cases:
        if P > F:
            P = F
        q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, D, F, G)
        pq, pk = mod.feature_map(q, Wq, bq, P), mod.feature_map(k, Wk, bk, P)
        got = mod.hybrid_attention_quadratic(q, k, v, pq, pk, L, Tc, To)
        want = mod.hybrid_attention_bruteforce(q, k, v, Wq, bq, Wk, bk, P, L, Tc, To)
        np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12,
                                   err_msg=f"T={T} L={L} Tc={Tc} To={To} P={P}")


def check_recurrent_and_streaming(mod):
    rng = np.random.default_rng(5)
    for (T, L, Tc, To, P) in [(7, 4, 3, 1, 2), (8, 3, 2, 0, 1), (9, 2, 1, 3, 3), (5, 5, 5, 2, 2),
                              (11, 3, 3, 2, 2), (4, 6, 1, 0, 2)]:
        q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, 8, 8, 2)
        pq, pk = mod.feature_map(q, Wq, bq, P), mod.feature_map(k, Wk, bk, P)
        quad = mod.hybrid_attention_quadratic(q, k, v, pq, pk, L, Tc, To)
        rec, S_seen, Z_seen = mod.hybrid_attention_recurrent(q, k, v, pq, pk, L, Tc, To,
                                                             return_states=True)
        np.testing.assert_allclose(rec, quad, rtol=1e-12, atol=1e-12)
        S_cf, Z_cf = mod.prefix_states(k, v, Wk, bk, P, L, Tc, To)
        np.testing.assert_allclose(np.stack(S_seen), S_cf, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(np.stack(Z_seen), Z_cf, rtol=1e-12, atol=1e-12)
        # streaming: chunk by chunk, keeping only (S, Z) and the last To frames
        S = np.zeros((pk.shape[1], v.shape[1])); Z = np.zeros(pk.shape[1])
        outs = []
        for (w, s, e) in mod.chunk_bounds(T, Tc, To):
            o, S, Z = mod.chunk_forward(q[s * L:e * L], k[w * L:e * L], v[w * L:e * L], Wq, bq,
                                        Wk, bk, P, S, Z, L, s, e - s, To)
            outs.append(o)
        np.testing.assert_allclose(np.concatenate(outs), quad, rtol=1e-12, atol=1e-12)
        m = max(0, T - To) * L
        np.testing.assert_allclose(S, pk[:m].T @ v[:m], rtol=1e-12, atol=1e-12)


def check_invariants(mod):
    rng = np.random.default_rng(6)
    T, L, Tc, To = 7, 4, 3, 1
    q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, 8, 8, 2, kscale=2.0)
    pq, pk = mod.feature_map(q, Wq, bq, 2), mod.feature_map(k, Wk, bk, 2)
    out = mod.hybrid_attention_quadratic(q, k, v, pq, pk, L, Tc, To)
    # convex combination of the visible values (every weight is positive)
    for i in range(T * L):
        e = min(((i // L) // Tc + 1) * Tc, T) * L
        assert np.all(out[i] <= v[:e].max(axis=0) + 1e-12)
        assert np.all(out[i] >= v[:e].min(axis=0) - 1e-12)
    # constant values give the constant back
    vc = np.tile(rng.standard_normal((1, 8)), (T * L, 1))
    np.testing.assert_allclose(mod.hybrid_attention_quadratic(q, k, vc, pq, pk, L, Tc, To), vc,
                               rtol=1e-12, atol=1e-12)
    # jointly permuting the (k, v) tokens inside one frame changes nothing
    perm = np.arange(T * L)
    f = 2
    perm[f * L:(f + 1) * L] = f * L + rng.permutation(L)
    out_p = mod.hybrid_attention_quadratic(q, k[perm], v[perm], pq, pk[perm], L, Tc, To)
    np.testing.assert_allclose(out_p, out, rtol=1e-12, atol=1e-12)


def check_rows_form(mod):
    rng = np.random.default_rng(7)
    for (T, L, Tc, To, P) in [(7, 5, 3, 1, 2), (5, 4, 1, 2, 3)]:
        q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, 8, 8, 2)
        pq, pk = mod.feature_map(q, Wq, bq, P), mod.feature_map(k, Wk, bk, P)
        quad = mod.hybrid_attention_quadratic(q, k, v, pq, pk, L, Tc, To)
        rows = np.array([0, 3, L * Tc, T * L - 1, (T * L) // 2])
        got = mod.hybrid_attention_rows(q, k, v, Wq, bq, Wk, bk, P, L, Tc, To, rows)
        np.testing.assert_allclose(got, quad[rows], rtol=1e-12, atol=1e-12)


def check_elu1_featmap(mod):
    """kind "elu1" with identity weights (G = D groups of 1 x 1) and no bias is elu(x) + 1 of the
    raw token, as in the linear attention of ReHyAt overview §2.1.2; with general weights it is
    elu(u) + 1 of the same grouped linear u as the polynomial map."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((40, 16)) * 2.0
    eye = np.ones((16, 1, 1))
    got = mod.feature_map(x, eye, None, 1, mod.PHI_ELU1)
    want = (torch.nn.functional.elu(torch.from_numpy(x)) + 1.0).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-15)
    _, _, _, W, b, _, _ = _rand_problem(rng, 1, 1, 16, 8, 4, bias=0.3)
    u = torch.nn.functional.conv1d(torch.from_numpy(x).T[None], torch.from_numpy(W).reshape(8, 4, 1),
                                   bias=torch.from_numpy(b), groups=4)[0].T
    want = (torch.nn.functional.elu(u) + 1.0).numpy()
    np.testing.assert_allclose(mod.feature_map(x, W, b, 3, mod.PHI_ELU1), want, rtol=1e-13, atol=1e-14)


def check_elu1_hybrid(mod):
    """With phi = elu + 1: one chunk with no window is the pages' linear attention
    phi(Q) (phi(K)^T V) normalised; the chunked hybrid matches the scalar brute force."""
    rng = np.random.default_rng(12)
    T, L, D = 4, 3, 8
    q, k, v, _, _, _, _ = _rand_problem(rng, T, L, D, 8, 2)
    eye = np.ones((D, 1, 1))
    pq, pk = mod.feature_map(q, eye, None, 1, mod.PHI_ELU1), mod.feature_map(k, eye, None, 1, mod.PHI_ELU1)
    M = np.full((T, T), mod.SET_LINEAR, dtype=np.int8)
    got = mod.hybrid_attention_masked(q, k, v, pq, pk, L, M)
    eq = np.where(q > 0, q + 1, np.exp(q)); ek = np.where(k > 0, k + 1, np.exp(k))
    want = (eq @ (ek.T @ v)) / (eq @ ek.sum(axis=0))[:, None]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    for (T, L, Tc, To) in [(6, 2, 2, 1), (5, 3, 3, 0), (7, 1, 1, 2)]:
        q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, 4, 4, 2, bias=0.2)
        pq = mod.feature_map(q, Wq, bq, 1, mod.PHI_ELU1)
        pk = mod.feature_map(k, Wk, bk, 1, mod.PHI_ELU1)
        quad = mod.hybrid_attention_quadratic(q, k, v, pq, pk, L, Tc, To)
        brute = mod.hybrid_attention_bruteforce(q, k, v, Wq, bq, Wk, bk, 1, L, Tc, To, mod.PHI_ELU1)
        np.testing.assert_allclose(quad, brute, rtol=1e-11, atol=1e-12)


def check_variable_schedule(mod):
    """A variable schedule (longer first chunk, per-chunk overlap) streamed with the recurrent
    step, each call folding what the next chunk's window no longer holds, equals the quadratic
    form under the schedule's frame mask; a uniform schedule gives the standard mask."""
    rng = np.random.default_rng(13)
    assert (mod.schedule_mask(mod.schedule_bounds([3, 3, 3, 1], [1, 1, 1, 1]))
            == mod.rehyat_mask(10, 3, 1)).all()
    L = 2
    for cfs, ovs in [([5, 3, 3, 2], [0, 1, 2, 1]), ([1, 2, 4, 1, 3], [0, 1, 2, 2, 1]),
                     ([4, 4], [0, 4])]:
        T = sum(cfs)
        q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, T, L, 8, 8, 2, bias=0.1)
        pq, pk = mod.feature_map(q, Wq, bq, 2), mod.feature_map(k, Wk, bk, 2)
        bounds = mod.schedule_bounds(cfs, ovs)
        want = mod.hybrid_attention_masked(q, k, v, pq, pk, L, mod.schedule_mask(bounds))
        S, Z = np.zeros((8, 8)), np.zeros(8)
        got = []
        for c, (w, s0, e) in enumerate(bounds):
            nxt = ovs[c + 1] if c + 1 < len(ovs) else ovs[c]
            o, S, Z = mod.chunk_forward(q[s0 * L:e * L], k[w * L:e * L], v[w * L:e * L], Wq, bq,
                                        Wk, bk, 2, S, Z, L, s0, e - s0, ovs[c], To_next=nxt)
            got.append(o)
        np.testing.assert_allclose(np.concatenate(got), want, rtol=1e-12, atol=1e-12)
    # a next overlap reaching past the current window needs frames already folded: refused
    q, k, v, Wq, bq, Wk, bk = _rand_problem(rng, 4, L, 8, 8, 2)
    with pytest.raises(ValueError):
        mod.chunk_forward(q[2 * L:3 * L], k[L:3 * L], v[L:3 * L], Wq, bq, Wk, bk, 2, np.zeros((8, 8)),
                          np.zeros(8), L, 2, 1, 1, To_next=3)


PINS = [check_rows_form, check_golden, check_featmap_conv1d, check_single_chunk_is_softmax, check_linear_only,
        check_bruteforce, check_recurrent_and_streaming, check_invariants, check_elu1_featmap,
        check_elu1_hybrid, check_variable_schedule]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(O)


def test_windows_of_the_tiny_workload():
    # 6 frames, Tc=3, To=1: chunk 0 owns frames 0-2 (window 0-2), chunk 1 owns 3-5 (window 2-5)
    assert O.chunk_bounds(6, 3, 1) == [(0, 0, 3), (2, 3, 6)]
    # ragged 41-frame case: 14 chunks, the last owns frames 39-40 and sees frames 38-40
    b = O.chunk_bounds(41, 3, 1)
    assert len(b) == 14 and b[-1] == (38, 39, 41)
    assert O.part_sizes(128, 3) == [43, 43, 42]


# ------------------------------------------------------------------------------------------
# mutation test: plausible mistakes planted in a copy of the oracle must fail some pin
# ------------------------------------------------------------------------------------------

MUTATIONS = [
    ("linear term without the e^-mu shift",
     "weights[:, li] = (phi_q[rows] @ phi_k[li].T) * np.exp(-mu)",
     "weights[:, li] = (phi_q[rows] @ phi_k[li].T)"),
    ("part powers reversed", "softplus(u[:, start:start + size]) ** p",
     "softplus(u[:, start:start + size]) ** (len(part_sizes(F, P)) - p + 1)"),
    ("grouped weight transposed", "x[:, g * Dg:(g + 1) * Dg] @ W[g].T",
     "x[:, g * Dg:(g + 1) * Dg] @ W[g]"),
    ("overlap one frame too wide", "w = max(0, s - To)\n", "w = max(0, s - To - 1)\n"),
    ("logits scaled by 1/D", "logits = q[rows] @ k[sm].T / math.sqrt(D)",
     "logits = q[rows] @ k[sm].T / D"),
    ("softplus without the log1p", "np.log1p(np.exp(-np.abs(x)))", "np.exp(-np.abs(x))"),
    ("recurrent fold starts at the chunk, not the window",
     "dep = slice(w * L, w_next * L)", "dep = slice(s * L, w_next * L)"),
    ("bias dropped", "u = u + np.asarray(bias, dtype=np.float64)[None, :]", "u = u"),
    ("linear normaliser dropped in the recurrent form",
     "den = den + shift * (phi_q_c @ Z)[:, None]", "den = den"),
    ("elu + 1 linear for negative inputs", "np.where(u > 0, u + 1.0, np.exp(np.minimum(u, 0.0)))",
     "np.where(u > 0, u + 1.0, u + 1.0)"),
    ("elu + 1 without the + 1", "np.where(u > 0, u + 1.0, np.exp(np.minimum(u, 0.0)))",
     "np.where(u > 0, u, np.exp(np.minimum(u, 0.0)) - 1.0)"),
    ("streaming fold ignores the next chunk's overlap",
     "w_next = max(0, frames_before + chunk_frames - To_next)",
     "w_next = max(0, frames_before + chunk_frames - To)"),
    ("streaming fold uses the chunk's own To twice",
     "w_next = max(0, frames_before + chunk_frames - To_next)",
     "w_next = max(0, frames_before + chunk_frames - 2 * To_next)"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(desc, old, new):
    src = open(O.__file__).read()
    assert src.count(old) == 1, f"mutation anchor not unique for: {desc}"
    mod = types.ModuleType("mutant")
    exec(compile(src.replace(old, new), "mutant", "exec"), mod.__dict__)
    failed = []
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError, pytest.fail.Exception):
            failed.append(pin.__name__)
    assert failed, f"no pin caught: {desc}"
