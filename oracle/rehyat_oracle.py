"""Float64 CPU oracle for ReHyAt chunk-wise recurrent hybrid attention (forward pass).

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously-correct statement of what
the hybrid attention forward computes.  Only the tests, the smoke check and the CPU-baseline leg
of the benchmark may import it; the CUDA library never does, and this module imports nothing
from the CUDA path.  Every routine works in float64 NumPy on whatever values it is given (bf16
tensors are upcast by the caller, so the oracle sees exactly the numbers the GPU sees).

Sources (page titles and sections):

* "ReHyAt overview" page (maplevalley.com.cn, news 2180822):
  - §2.1.1 softmax attention, exp(q.k / sqrt(D)) kernel;
  - §2.1.2 linear attention phi_Q (phi_K^T V) (printed without its normaliser);
  - §2.2.1 the hybrid split into a softmax region T_S (current temporal chunk and its
    neighbourhood) and a linear region T_L (everything else), joined as
    (softmax part + linear part) / (softmax normaliser + linear normaliser); chunks of Tc
    frames (typ. 3) with an overlap of To frames (typ. 1);
  - §2.2.2 the polynomial feature map: grouped 1x1 linear, split into P parts, part p raised
    to power p, concatenated;
  - §2.3 causal chunk recurrence with the states S = sum phi_K v^T and Z = sum phi_K,
    S_{t+1} = S_t + sum(phi_K v^T), Z_{t+1} = Z_t + sum(phi_K);
  - §5.2 the streaming generation loop (output, states) = block(chunk, states).
* "Neuer Ansatz zur effizienten Videogenerierung mit ReHyAt" (mind-verse.de), sections
  "Temporär segmentierte hybride Aufmerksamkeit" (softmax inside overlapping chunks, linear
  for all other tokens) and "Rekurrente Formulierung und konstante Speichernutzung".

Readings where the pages are silent (each one is listed with its reason in the design notes):

* Inside a chunk and its overlap the softmax is bidirectional; only later chunks are masked.
* The overlap frames are the To frames *before* the chunk; queries belong to exactly one chunk.
* The frames folded into (S, Z) after chunk c are the ones that leave the softmax window,
  frames [w_c, w_{c+1}) with w_c = max(0, c*Tc - To).
* The linear branch keeps its normaliser phi_q . Z (the §2.1.2 listing drops it, §2.2.1 keeps it).
* The feature-map activation is softplus; part p (1-based) of the split gets power p; when P
  does not divide F the parts have the sizes numpy.array_split gives.
* The logit scale 1/sqrt(D) applies to the softmax logits only, never to phi.

Every function here is a direct transcription of a definition; none of it is blocked, fused or
reordered beyond what the definition states.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "softplus",
    "part_sizes",
    "feature_map",
    "elu1",
    "PHI_POLY",
    "PHI_ELU1",
    "chunk_bounds",
    "rehyat_mask",
    "schedule_bounds",
    "schedule_mask",
    "hybrid_attention_masked",
    "hybrid_attention_quadratic",
    "hybrid_attention_recurrent",
    "chunk_forward",
    "prefix_states",
    "hybrid_attention_bruteforce",
    "hybrid_attention_rows",
    "SET_SOFTMAX",
    "SET_LINEAR",
    "SET_NONE",
]

SET_NONE = 0      # key frame invisible to the query frame (future chunk)
SET_SOFTMAX = 1   # key frame in T_S: exact exp(q.k/sqrt(D)) weight
SET_LINEAR = 2    # key frame in T_L: phi_q(q) . phi_k(k) weight


# ---------------------------------------------------------------------------------------------
# Feature map (ReHyAt overview §2.2.2; separate phi_q and phi_k per §3.1.1)
# ---------------------------------------------------------------------------------------------

def softplus(x: np.ndarray) -> np.ndarray:
    """log(1 + e^x), written in the overflow-free form max(x, 0) + log1p(e^{-|x|})."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def part_sizes(F: int, P: int) -> list[int]:
    """Sizes of the P contiguous parts the F features are split into (numpy.array_split order:
    the first F mod P parts are one longer)."""
    if P < 1 or F < P:
        raise ValueError(f"need 1 <= P <= F, got P={P}, F={F}")
    base, extra = divmod(F, P)
    return [base + 1 if p < extra else base for p in range(P)]


PHI_POLY = "poly"   # softplus parts raised to powers 1..P (ReHyAt overview §2.2.2)
PHI_ELU1 = "elu1"   # elu(u) + 1, the linear-attention feature map of ReHyAt overview §2.1.2


def elu1(u: np.ndarray) -> np.ndarray:
    """elu(u) + 1: u + 1 for u > 0, e^u otherwise (continuous at 0, always > 0)."""
    u = np.asarray(u, dtype=np.float64)
    return np.where(u > 0, u + 1.0, np.exp(np.minimum(u, 0.0)))


def feature_map(x: np.ndarray, W: np.ndarray, bias: np.ndarray | None, P: int,
                kind: str = PHI_POLY) -> np.ndarray:
    """Feature map phi(x): the polynomial map of ReHyAt overview §2.2.2 (kind "poly"), or the
    elu(.) + 1 map of the linear attention in §2.1.2 (kind "elu1") applied after the same
    grouped linear; with identity weights (G = D, W all ones, no bias) "elu1" is elu(x) + 1 of
    the raw token, as printed there.

    x    : [n, D] tokens of one head.
    W    : [G, F/G, D/G] weights of the grouped 1x1 linear ("light MLP of grouped 1x1 convs"):
           group g maps input features [g*D/G, (g+1)*D/G) to output features
           [g*F/G, (g+1)*F/G) as u_g = x_g W[g]^T.
    bias : [F] or None.
    P    : number of parts; part p (1-based) of u is mapped to softplus(u_p) ** p, and the parts
           are concatenated back in order (kind "poly"; ignored for "elu1").
    Returns phi [n, F], every entry > 0.
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    n, D = x.shape
    G, Fg, Dg = W.shape
    if G * Dg != D:
        raise ValueError("W does not match D")
    F = G * Fg
    u = np.empty((n, F), dtype=np.float64)
    for g in range(G):
        u[:, g * Fg:(g + 1) * Fg] = x[:, g * Dg:(g + 1) * Dg] @ W[g].T
    if bias is not None:
        u = u + np.asarray(bias, dtype=np.float64)[None, :]
    if kind == PHI_ELU1:
        return elu1(u)
    if kind != PHI_POLY:
        raise ValueError(f"unknown feature map kind {kind!r}")
    out = np.empty_like(u)
    start = 0
    for p, size in enumerate(part_sizes(F, P), start=1):
        out[:, start:start + size] = softplus(u[:, start:start + size]) ** p
        start += size
    return out


# ---------------------------------------------------------------------------------------------
# Chunk schedule (ReHyAt overview §2.2.1, §2.3)
# ---------------------------------------------------------------------------------------------

def chunk_bounds(T: int, Tc: int, To: int) -> list[tuple[int, int, int]]:
    """For every temporal chunk c return (w_c, s_c, e_c) in frames: the chunk owns query frames
    [s_c, e_c) = [c*Tc, min((c+1)*Tc, T)); its softmax window is key frames [w_c, e_c) with
    w_c = max(0, c*Tc - To); key frames [0, w_c) are its linear region."""
    if T < 1 or Tc < 1 or To < 0:
        raise ValueError("need T >= 1, Tc >= 1, To >= 0")
    out = []
    for c in range(-(-T // Tc)):
        s = c * Tc
        e = min(s + Tc, T)
        w = max(0, s - To)
        out.append((w, s, e))
    return out


def schedule_bounds(chunk_frames, overlaps) -> list[tuple[int, int, int]]:
    """(w_c, s_c, e_c) of a variable schedule (ReHyAt overview §5.2: a longer chunk for key
    frames such as the first, more overlap where motion is strong): chunk c owns the next
    chunk_frames[c] frames and its softmax window reaches overlaps[c] frames back."""
    if len(chunk_frames) != len(overlaps) or not chunk_frames:
        raise ValueError("one overlap per chunk")
    out, s = [], 0
    for cf, o in zip(chunk_frames, overlaps):
        if cf < 1 or o < 0:
            raise ValueError("need chunk_frames >= 1 and overlaps >= 0")
        out.append((max(0, s - o), s, s + cf))
        s += cf
    return out


def schedule_mask(bounds) -> np.ndarray:
    """Frame-level set assignment of any chunk schedule given as (w_c, s_c, e_c) triples."""
    T = bounds[-1][2]
    M = np.full((T, T), SET_NONE, dtype=np.int8)
    for (w, s, e) in bounds:
        M[s:e, w:e] = SET_SOFTMAX
        M[s:e, 0:w] = SET_LINEAR
    return M


def rehyat_mask(T: int, Tc: int, To: int) -> np.ndarray:
    """Frame-level set assignment M[query_frame, key_frame] of the standard ReHyAt pattern."""
    M = np.full((T, T), SET_NONE, dtype=np.int8)
    for (w, s, e) in chunk_bounds(T, Tc, To):
        M[s:e, w:e] = SET_SOFTMAX
        M[s:e, 0:w] = SET_LINEAR
    return M


# ---------------------------------------------------------------------------------------------
# Quadratic (non-recurrent) form: the output formula of §2.2.1 evaluated key by key
# ---------------------------------------------------------------------------------------------

def hybrid_attention_masked(q, k, v, phi_q, phi_k, frame_tokens: int, M: np.ndarray) -> np.ndarray:
    """out_i = (sum_{j in T_S(i)} e^{s_ij} v_j + sum_{j in T_L(i)} (phi_q_i . phi_k_j) v_j)
             / (sum_{j in T_S(i)} e^{s_ij}     + sum_{j in T_L(i)} (phi_q_i . phi_k_j)),
    s_ij = q_i . k_j / sqrt(D), with the sets given frame by frame by M (any assignment, so that
    T_S = all and T_S = empty can be expressed).  The weights of every key are materialised
    explicitly.  A per-row shift mu (the row max over T_S, or 0 when T_S is empty) is taken out
    of the exponentials and the linear weights alike, so it cancels exactly in the ratio.
    Rows whose query frame sees no key at all are returned as NaN."""
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    phi_q = np.asarray(phi_q, np.float64); phi_k = np.asarray(phi_k, np.float64)
    n, D = q.shape
    L = frame_tokens
    T = n // L
    if T * L != n or M.shape != (T, T):
        raise ValueError("token count is not frames x frame_tokens, or mask shape is wrong")
    key_frame = np.arange(n) // L
    out = np.full((n, v.shape[1]), np.nan, dtype=np.float64)
    for tq in range(T):
        rows = slice(tq * L, (tq + 1) * L)
        sm = M[tq][key_frame] == SET_SOFTMAX
        li = M[tq][key_frame] == SET_LINEAR
        if not (sm.any() or li.any()):
            continue
        weights = np.zeros((L, n), dtype=np.float64)
        if sm.any():
            logits = q[rows] @ k[sm].T / math.sqrt(D)
            mu = logits.max(axis=1, keepdims=True)
            weights[:, sm] = np.exp(logits - mu)
        else:
            mu = np.zeros((L, 1))
        if li.any():
            weights[:, li] = (phi_q[rows] @ phi_k[li].T) * np.exp(-mu)
        out[rows] = (weights @ v) / weights.sum(axis=1, keepdims=True)
    return out


def hybrid_attention_quadratic(q, k, v, phi_q, phi_k, frame_tokens: int, Tc: int, To: int):
    """The ReHyAt hybrid output for the standard chunk pattern, quadratic form."""
    T = q.shape[0] // frame_tokens
    return hybrid_attention_masked(q, k, v, phi_q, phi_k, frame_tokens, rehyat_mask(T, Tc, To))


def hybrid_attention_rows(q, k, v, Wq, bq, Wk, bk, P: int, frame_tokens: int, Tc: int, To: int,
                          rows, kind: str = PHI_POLY) -> np.ndarray:
    """The quadratic form evaluated for selected query rows only (for sequences too long to
    evaluate whole): row i of chunk c = (i // L) // Tc weighs keys [w_c L, e_c L) by
    exp(q.k/sqrt(D)) and keys [0, w_c L) by phi_q(q).phi_k(k), shifted by the row max of the
    window logits, and divides by the sum of the weights."""
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    n, D = q.shape
    L = frame_tokens
    T = n // L
    bounds = chunk_bounds(T, Tc, To)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), v.shape[1]))
    phi_q = feature_map(q[rows], Wq, bq, P, kind)
    need = max(bounds[(int(r) // L) // Tc][0] for r in rows) * L
    phi_k = feature_map(k[:need], Wk, bk, P, kind) if need > 0 else None
    for a, r in enumerate(rows):
        w, s, e = bounds[(int(r) // L) // Tc]
        logits = k[w * L:e * L] @ q[r] / math.sqrt(D)
        mu = logits.max()
        ws = np.exp(logits - mu)
        num = ws @ v[w * L:e * L]
        den = ws.sum()
        if w > 0:
            wl = (phi_k[:w * L] @ phi_q[a]) * math.exp(-mu)
            num = num + wl @ v[:w * L]
            den = den + wl.sum()
        out[a] = num / den
    return out


# ---------------------------------------------------------------------------------------------
# Recurrent form: chunk by chunk with running states (ReHyAt overview §2.3)
# ---------------------------------------------------------------------------------------------

def _window_output(q_c, k_w, v_w, phi_q_c, S, Z, has_linear: bool):
    """Output rows of one chunk from its softmax window and the states, (A v + e^{-mu} phi_q S) /
    (A 1 + e^{-mu} phi_q Z) with A = e^{s - mu}, mu = row max of the window logits."""
    D = q_c.shape[1]
    logits = q_c @ k_w.T / math.sqrt(D)
    mu = logits.max(axis=1, keepdims=True)
    A = np.exp(logits - mu)
    num = A @ v_w
    den = A.sum(axis=1, keepdims=True)
    if has_linear:
        shift = np.exp(-mu)
        num = num + shift * (phi_q_c @ S)
        den = den + shift * (phi_q_c @ Z)[:, None]
    return num / den


def hybrid_attention_recurrent(q, k, v, phi_q, phi_k, frame_tokens: int, Tc: int, To: int,
                               return_states: bool = False):
    """Chunk-wise recurrent form.  S (F x D) and Z (F) start at zero; chunk c reads them, then the
    frames that leave the softmax window, [w_c, w_{c+1}), are folded in:
    S <- S + sum phi_k(k) v^T,  Z <- Z + sum phi_k(k).
    With return_states the states each chunk read are returned as lists as well."""
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    phi_q = np.asarray(phi_q, np.float64); phi_k = np.asarray(phi_k, np.float64)
    n = q.shape[0]
    L = frame_tokens
    T = n // L
    bounds = chunk_bounds(T, Tc, To)
    F, Dv = phi_k.shape[1], v.shape[1]
    S = np.zeros((F, Dv)); Z = np.zeros(F)
    out = np.empty((n, Dv))
    S_seen, Z_seen = [], []
    for c, (w, s, e) in enumerate(bounds):
        S_seen.append(S.copy()); Z_seen.append(Z.copy())
        rows = slice(s * L, e * L)
        win = slice(w * L, e * L)
        out[rows] = _window_output(q[rows], k[win], v[win], phi_q[rows], S, Z, has_linear=w > 0)
        if c + 1 < len(bounds):
            w_next = bounds[c + 1][0]
            dep = slice(w * L, w_next * L)
            S = S + phi_k[dep].T @ v[dep]
            Z = Z + phi_k[dep].sum(axis=0)
    if return_states:
        return out, S_seen, Z_seen
    return out


def prefix_states(k, v, Wk, bk, P: int, frame_tokens: int, Tc: int, To: int,
                  kind: str = PHI_POLY):
    """Closed form of the state every chunk reads: S_c = phi_k[0:w_c]^T V[0:w_c],
    Z_c = phi_k[0:w_c]^T 1 (the linear region of chunk c, summed directly)."""
    phi_k = feature_map(k, Wk, bk, P, kind)
    v = np.asarray(v, np.float64)
    T = k.shape[0] // frame_tokens
    Ss, Zs = [], []
    for (w, s, e) in chunk_bounds(T, Tc, To):
        m = w * frame_tokens
        Ss.append(phi_k[:m].T @ v[:m])
        Zs.append(phi_k[:m].sum(axis=0))
    return np.stack(Ss), np.stack(Zs)


def chunk_forward(q_c, k_win, v_win, Wq, bq, Wk, bk, P: int, S, Z, frame_tokens: int,
                  frames_before: int, chunk_frames: int, To: int, kind: str = PHI_POLY,
                  To_next: int | None = None):
    """One streaming step (ReHyAt overview §5.2 loop, states per §2.3).

    q_c   : [chunk_frames*L, D] queries of the chunk that starts at frame `frames_before`.
    k_win, v_win : [(o + chunk_frames)*L, D] with o = min(To, frames_before): the overlap frames
            followed by the chunk's own frames (the softmax window).
    S, Z  : states holding every frame before the window.
    Returns (out, S_new, Z_new).  After the output is formed, the window frames that the next
    chunk no longer sees, [w_c, w_{c+1}) with w_{c+1} = max(0, frames_before + chunk_frames -
    To_next), are folded into the returned states; To_next is the next chunk's overlap (the
    same To unless the schedule varies it)."""
    L = frame_tokens
    o = min(To, frames_before)
    w = frames_before - o
    if k_win.shape[0] != (o + chunk_frames) * L or q_c.shape[0] != chunk_frames * L:
        raise ValueError("window or chunk size does not match frames_before/chunk_frames/To")
    phi_q = feature_map(q_c, Wq, bq, P, kind)
    phi_k = feature_map(k_win, Wk, bk, P, kind)
    out = _window_output(np.asarray(q_c, np.float64), np.asarray(k_win, np.float64),
                         np.asarray(v_win, np.float64), phi_q, np.asarray(S, np.float64),
                         np.asarray(Z, np.float64), has_linear=w > 0)
    if To_next is None:
        To_next = To
    w_next = max(0, frames_before + chunk_frames - To_next)
    if w_next < w:
        raise ValueError("the next chunk's overlap reaches frames already folded into S")
    nd = (w_next - w) * L
    S_new = np.asarray(S, np.float64) + phi_k[:nd].T @ np.asarray(v_win, np.float64)[:nd]
    Z_new = np.asarray(Z, np.float64) + phi_k[:nd].sum(axis=0)
    return out, S_new, Z_new


# ---------------------------------------------------------------------------------------------
# Brute force: one scalar term per (query, key) pair, for tiny inputs only
# ---------------------------------------------------------------------------------------------

def hybrid_attention_bruteforce(q, k, v, Wq, bq, Wk, bk, P: int, frame_tokens: int, Tc: int,
                                To: int, kind: str = PHI_POLY) -> np.ndarray:
    """Pure-Python loops.  For every query token i (frame t_i, chunk c = t_i // Tc) and every key
    token j (frame t_j): future chunks (t_j >= end of chunk c) are skipped; frames inside
    [max(0, c*Tc - To), end of chunk c) contribute exp(q.k/sqrt(D)); earlier frames contribute
    phi_q(q_i).phi_k(k_j), phi evaluated scalar by scalar.  No shift is used, so this is only for
    inputs whose logits stay well inside the float64 exponent range."""
    q = [[float(a) for a in row] for row in np.asarray(q, np.float64)]
    k = [[float(a) for a in row] for row in np.asarray(k, np.float64)]
    v = [[float(a) for a in row] for row in np.asarray(v, np.float64)]
    n, D, Dv = len(q), len(q[0]), len(v[0])
    T = n // frame_tokens

    def phi(x, W, b):
        G, Fg, Dg = np.asarray(W).shape
        F = G * Fg
        u = []
        for f in range(F):
            g, r = divmod(f, Fg)
            acc = 0.0 if b is None else float(b[f])
            for d in range(Dg):
                acc += float(W[g][r][d]) * x[g * Dg + d]
            u.append(acc)
        if kind == PHI_ELU1:
            return [a + 1.0 if a > 0 else math.exp(a) for a in u]
        res, f = [], 0
        for p, size in enumerate(part_sizes(F, P), start=1):
            for _ in range(size):
                sp = math.log1p(math.exp(u[f])) if u[f] < 30 else u[f] + math.log1p(math.exp(-u[f]))
                res.append(sp ** p)
                f += 1
        return res

    pq = [phi(row, Wq, bq) for row in q]
    pk = [phi(row, Wk, bk) for row in k]
    out = []
    for i in range(n):
        c = (i // frame_tokens) // Tc
        end = min((c + 1) * Tc, T)
        win = max(0, c * Tc - To)
        num = [0.0] * Dv
        den = 0.0
        for j in range(n):
            tj = j // frame_tokens
            if tj >= end:
                continue
            if tj >= win:
                wgt = math.exp(sum(q[i][d] * k[j][d] for d in range(D)) / math.sqrt(D))
            else:
                wgt = sum(a * b for a, b in zip(pq[i], pk[j]))
            den += wgt
            for d in range(Dv):
                num[d] += wgt * v[j][d]
        out.append([x / den for x in num])
    return np.array(out, dtype=np.float64)
