"""Thin ctypes binding of librehyat.so (C ABI in include/rehyat.h).

Argument marshalling only: tensors are checked for device/dtype/shape/contiguity, outputs and
workspaces are allocated with torch on the tensors' device, and every computation runs in the
library's CUDA kernels.  There is no CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "librehyat.so")

REHYAT_F32 = 0
REHYAT_BF16 = 1
PHI_POLY = 0   # softplus parts raised to powers 1..P
PHI_ELU1 = 1   # elu(u) + 1

STATUS = {0: "OK", -1: "ERR_ARG", -2: "ERR_SHAPE", -3: "ERR_DTYPE", -4: "ERR_WORKSPACE",
          -5: "ERR_CUDA", -6: "ERR_TIMEOUT", -7: "ERR_ALIGN", -8: "ERR_BOUNDS"}

EXPORTED = ["rehyat_last_error", "rehyat_version", "rehyat_featmap",
            "rehyat_forward_workspace_size", "rehyat_forward", "rehyat_forward_states",
            "rehyat_forward_phiq", "rehyat_forward_attend", "rehyat_chunk_workspace_size",
            "rehyat_chunk_forward", "rehyat_chunk_forward_sched", "rehyat_chunk_carry_workspace_size",
            "rehyat_chunk_forward_carry", "rehyat_chunk_forward_static", "rehyat_chunk_states",
            "rehyat_forward_train", "rehyat_backward_workspace_size", "rehyat_backward",
            "rehyat_gemm_bf16", "rehyat_segment_workspace_size", "rehyat_segment_states",
            "rehyat_segment_attend", "rehyat_selftest_wait_timeout", "rehyat_selftest_bounds",
            "rehyat_sync_status", "rehyat_debug_bounds"]


class RehyatError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int), ("F", ctypes.c_int),
                ("G", ctypes.c_int), ("P", ctypes.c_int), ("phi", ctypes.c_int)]


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def use_library(path: str) -> ctypes.CDLL:
    """Make every later call go through the library at `path` (for example the debug-bounds
    build, build.build(debug_bounds=True)); returns it loaded."""
    global _lib, _LIB_PATH
    _lib, _LIB_PATH = None, path
    return load()


def load() -> ctypes.CDLL:
    """Load librehyat.so (built in-tree by the package build step) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"librehyat.so is not built ({_LIB_PATH}); run the package build "
                           "step (hybrid_softmax_linear_chunked_b200.build.build()) first")
    L = ctypes.CDLL(_LIB_PATH)
    c_int, c_void_p, c_size_t = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    P = c_void_p
    L.rehyat_last_error.restype = ctypes.c_char_p
    L.rehyat_last_error.argtypes = []
    L.rehyat_version.restype = c_int
    L.rehyat_featmap.argtypes = [Dims, c_int, c_int, P, P, P, P, P]
    L.rehyat_forward_workspace_size.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int,
                                                ctypes.POINTER(c_size_t)]
    L.rehyat_forward.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P, P, P, P, P,
                                 P, c_size_t, P]
    L.rehyat_forward_states.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P, P,
                                        c_size_t, P]
    L.rehyat_forward_phiq.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P,
                                      c_size_t, P]
    L.rehyat_forward_attend.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P, P,
                                        c_size_t, P]
    L.rehyat_chunk_workspace_size.argtypes = [Dims, c_int, c_int, c_int, c_int,
                                              ctypes.POINTER(c_size_t)]
    L.rehyat_segment_workspace_size.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, c_int,
                                                c_int, ctypes.POINTER(c_size_t)]
    L.rehyat_segment_states.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                        P, P, P, P, P, P, P, c_size_t, P]
    L.rehyat_segment_attend.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                        P, P, P, P, P, c_int, P, P, P, P, c_size_t, P]
    L.rehyat_chunk_forward.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P, P, P,
                                       P, P, P, P, P, c_size_t, P]
    L.rehyat_chunk_forward_sched.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, c_int, P, P,
                                             P, P, P, P, P, P, P, P, P, c_size_t, P]
    L.rehyat_chunk_carry_workspace_size.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int,
                                                    ctypes.POINTER(c_size_t)]
    L.rehyat_chunk_forward_carry.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                             P, P, P, P, P, P, P, P, P, P, P, P, P, c_size_t, P]
    L.rehyat_chunk_forward_static.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P,
                                              P, P, P, P, P, P, P]
    L.rehyat_chunk_states.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P, P, P,
                                      P, c_size_t, P]
    LL = ctypes.c_longlong
    L.rehyat_forward_train.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int, P, P, P, P, P, P,
                                       P, P, P, P, c_size_t, P]
    L.rehyat_backward_workspace_size.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int,
                                                 ctypes.POINTER(c_size_t)]
    L.rehyat_backward.argtypes = [Dims, c_int, c_int, c_int, c_int, c_int] + [P] * 18 + [c_size_t, P]
    L.rehyat_gemm_bf16.argtypes = [c_int, c_int, c_int, c_int, P, LL, LL, c_int, P, LL, LL, c_int,
                                   P, LL, LL, c_int, c_int, ctypes.c_float, P]
    L.rehyat_selftest_wait_timeout.argtypes = [ctypes.c_longlong, P]
    L.rehyat_selftest_bounds.argtypes = [P, ctypes.c_longlong, ctypes.c_longlong, P]
    L.rehyat_debug_bounds.argtypes = []
    L.rehyat_sync_status.argtypes = [P]
    for name in EXPORTED:
        if name not in ("rehyat_last_error",):
            getattr(L, name).restype = c_int
    _lib = L
    return L


def _check(status: int) -> None:
    if status != 0:
        raise RehyatError(status, load().rehyat_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return REHYAT_BF16
    if t.dtype == torch.float32:
        return REHYAT_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dev(*ts: torch.Tensor) -> torch.device:
    dev = ts[0].device
    for t in ts:
        if t is None:
            continue
        if t.device.type != "cuda" or t.device != dev:
            raise ValueError("all tensors must be on the same CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return dev


def _shape(t: torch.Tensor | None, shape, what: str) -> None:
    """The library reads exactly the sizes the other arguments imply; a tensor of another shape
    is refused here, before anything is enqueued."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _frames(n_rows: int, frame_tokens: int, what: str) -> int:
    if frame_tokens < 1 or n_rows % frame_tokens:
        raise ValueError(f"{what}: {n_rows} rows are not a whole number of frames of "
                         f"{frame_tokens} tokens")
    return n_rows // frame_tokens


def _check_x_w(x: torch.Tensor, W: torch.Tensor, b: torch.Tensor | None, what: str) -> None:
    """x [B,H,n,D]; W [H,G,F/G,D/G]; b [H,F] or None."""
    if x.dim() != 4:
        raise ValueError(f"{what} must be [B,H,rows,D], got {tuple(x.shape)}")
    if W.dim() != 4 or W.shape[0] != x.shape[1] or W.shape[1] * W.shape[3] != x.shape[3]:
        raise ValueError(f"feature-map weights must be [H,G,F/G,D/G] for {what} of shape "
                         f"{tuple(x.shape)}, got {tuple(W.shape)}")
    _shape(b, (W.shape[0], W.shape[1] * W.shape[2]), "feature-map bias")


def _check_step(q, k, v, Wq, bq, Wk, bk, S, Z, out, frame_tokens: int, kv_frames: int | None,
                what_kv: str) -> int:
    """Shapes of a streaming step: q [B,H,cf*L,D]; k, v [B,H,kv_frames*L,D] (the chunk's own
    frames when kv_frames is None); S [B,H,F,D], Z [B,H,F]; out like q.  Returns cf."""
    _check_x_w(q, Wq, bq, "q")
    _check_x_w(q, Wk, bk, "q")
    _shape(Wk, Wq.shape, "Wk")
    cf = _frames(q.shape[2], frame_tokens, "q")
    B, H, _, D = q.shape
    F = Wq.shape[1] * Wq.shape[2]
    rows = (cf if kv_frames is None else kv_frames) * frame_tokens
    _shape(k, (B, H, rows, D), what_kv)
    _shape(v, (B, H, rows, D), what_kv.replace("k", "v", 1))
    _shape(S, (B, H, F, D), "S")
    _shape(Z, (B, H, F), "Z")
    _shape(out, q.shape, "out")
    return cf


def _weights(W: torch.Tensor, b: torch.Tensor | None):
    if W.dtype != torch.float32 or (b is not None and b.dtype != torch.float32):
        raise TypeError("feature-map weights and biases are fp32")
    return W, b


def dims_of(x: torch.Tensor, W: torch.Tensor, P: int, phi: int = 0) -> Dims:
    """Dims from x [B,H,n,D] and W [H,G,F/G,D/G]; phi is PHI_POLY or PHI_ELU1."""
    B, H, _, D = x.shape
    Hw, G, Fg, _ = W.shape
    if Hw != H:
        raise ValueError("W has a different head count than x")
    return Dims(B, H, D, G * Fg, G, P, phi)


def version() -> int:
    return load().rehyat_version()


def featmap(x: torch.Tensor, W: torch.Tensor, bias: torch.Tensor | None, P: int,
            phi: int = 0) -> torch.Tensor:
    """phi(x) for x [B,H,n,D] -> [B,H,n,F] (same dtype as x)."""
    L = load()
    dev = _dev(x, W, bias)
    _weights(W, bias)
    d = dims_of(x, W, P, phi)
    phi = torch.empty(x.shape[0], x.shape[1], x.shape[2], d.F, dtype=x.dtype, device=dev)
    _check(L.rehyat_featmap(d, _dtype_code(x), x.shape[2], _ptr(x), _ptr(W), _ptr(bias),
                            _ptr(phi), _stream(dev)))
    return phi


def forward_workspace_size(d: Dims, dtype_code: int, T: int, L_: int, Tc: int, To: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().rehyat_forward_workspace_size(d, dtype_code, T, L_, Tc, To, ctypes.byref(n)))
    return n.value


def chunk_workspace_size(d: Dims, dtype_code: int, L_: int, chunk_frames: int, To: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().rehyat_chunk_workspace_size(d, dtype_code, L_, chunk_frames, To,
                                              ctypes.byref(n)))
    return n.value


def _workspace(nbytes: int, dev: torch.device, workspace: torch.Tensor | None) -> torch.Tensor:
    if workspace is not None and workspace.numel() >= nbytes:
        return workspace
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)


def forward(q, k, v, Wq, bq, Wk, bk, *, P: int, phi: int = 0, frame_tokens: int, Tc: int, To: int,
            out: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Hybrid attention over a whole sequence: q, k, v [B,H,T*frame_tokens,D] -> out."""
    lib = load()
    _check_x_w(q, Wq, bq, "q")
    _check_x_w(q, Wk, bk, "q")
    _shape(Wk, Wq.shape, "Wk")
    for t, n in ((k, "k"), (v, "v"), (out, "out")):
        _shape(t, q.shape, n)
    dev = _dev(q, k, v, Wq, bq, Wk, bk)
    _weights(Wq, bq), _weights(Wk, bk)
    d = dims_of(q, Wq, P, phi)
    N = q.shape[2]
    if N % frame_tokens:
        raise ValueError("sequence length is not a multiple of frame_tokens")
    T = N // frame_tokens
    code = _dtype_code(q)
    ws = _workspace(forward_workspace_size(d, code, T, frame_tokens, Tc, To), dev, workspace)
    if out is None:
        out = torch.empty_like(q)
    _check(lib.rehyat_forward(d, code, T, frame_tokens, Tc, To, _ptr(q), _ptr(k), _ptr(v),
                              _ptr(Wq), _ptr(bq), _ptr(Wk), _ptr(bk), _ptr(out), _ptr(ws),
                              ws.numel(), _stream(dev)))
    return out


def segment_bounds(T: int, Tc: int, To: int, c0: int, c1: int) -> tuple[int, int, int]:
    """(s0, s1, h0) of the segment of chunks [c0, c1): query frames [s0, s1), key/value frames
    [h0, s1)."""
    s0, s1 = c0 * Tc, min(c1 * Tc, T)
    return s0, s1, max(0, s0 - To)


def segment_workspace_size(d: Dims, T: int, frame_tokens: int, Tc: int, To: int, c0: int,
                           c1: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().rehyat_segment_workspace_size(d, REHYAT_BF16, T, frame_tokens, Tc, To, c0, c1,
                                                ctypes.byref(n)))
    return n.value


def segment_states(k_seg, v_seg, Wk, bk, *, T: int, c0: int, c1: int, P: int, phi: int = 0,
                   frame_tokens: int, Tc: int, To: int, workspace: torch.Tensor,
                   S_seg: torch.Tensor | None = None, Z_seg: torch.Tensor | None = None):
    """First phase of a context-parallel segment (chunks [c0, c1) of a T-frame sequence):
    k_seg, v_seg [B,H,(s1-h0)*frame_tokens,D] bf16 (halo frames first).  Fills `workspace` with
    the segment's folds and returns their sum (S_seg [B,H,F,D], Z_seg [B,H,F] fp32)."""
    lib = load()
    _check_x_w(k_seg, Wk, bk, "k_seg")
    s0, s1, h0 = segment_bounds(T, Tc, To, c0, c1)
    B, H, _, D = k_seg.shape
    F = Wk.shape[1] * Wk.shape[2]
    _shape(k_seg, (B, H, (s1 - h0) * frame_tokens, D), "k_seg")
    _shape(v_seg, k_seg.shape, "v_seg")
    _shape(S_seg, (B, H, F, D), "S_seg")
    _shape(Z_seg, (B, H, F), "Z_seg")
    dev = _dev(k_seg, v_seg, Wk, bk, workspace)
    d = dims_of(k_seg, Wk, P, phi)
    B, H = d.B, d.H
    if S_seg is None:
        S_seg = torch.empty(B, H, d.F, d.D, dtype=torch.float32, device=dev)
    if Z_seg is None:
        Z_seg = torch.empty(B, H, d.F, dtype=torch.float32, device=dev)
    _dev(S_seg, Z_seg)
    _check(lib.rehyat_segment_states(d, _dtype_code(k_seg), T, frame_tokens, Tc, To, c0, c1,
                                     _ptr(k_seg), _ptr(v_seg), _ptr(Wk), _ptr(bk), _ptr(S_seg),
                                     _ptr(Z_seg), _ptr(workspace), workspace.numel(),
                                     _stream(dev)))
    return S_seg, Z_seg


def segment_attend(q_seg, k_seg, v_seg, Wq, bq, *, T: int, c0: int, c1: int, P: int,
                   phi: int = 0, frame_tokens: int, Tc: int, To: int, workspace: torch.Tensor,
                   S_prefix: torch.Tensor | None = None, Z_prefix: torch.Tensor | None = None,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """Second phase: the segment's outputs.  S_prefix [n,B,H,F,D] / Z_prefix [n,B,H,F] stack
    the segment sums of every earlier segment (None for the first)."""
    lib = load()
    _check_x_w(q_seg, Wq, bq, "q_seg")
    s0, s1, h0 = segment_bounds(T, Tc, To, c0, c1)
    B, H, _, D = q_seg.shape
    F = Wq.shape[1] * Wq.shape[2]
    _shape(q_seg, (B, H, (s1 - s0) * frame_tokens, D), "q_seg")
    _shape(k_seg, (B, H, (s1 - h0) * frame_tokens, D), "k_seg")
    _shape(v_seg, k_seg.shape, "v_seg")
    _shape(out, q_seg.shape, "out")
    if S_prefix is not None:
        _shape(S_prefix, (S_prefix.shape[0], B, H, F, D), "S_prefix")
    if Z_prefix is not None:
        _shape(Z_prefix, (Z_prefix.shape[0], B, H, F), "Z_prefix")
    dev = _dev(q_seg, k_seg, v_seg, Wq, bq, workspace)
    d = dims_of(q_seg, Wq, P, phi)
    n_prefix = 0
    if (S_prefix is None) != (Z_prefix is None):
        raise ValueError("give both S_prefix and Z_prefix or neither")
    if S_prefix is not None:
        _dev(S_prefix, Z_prefix)
        n_prefix = S_prefix.shape[0]
        if S_prefix.dtype != torch.float32 or Z_prefix.dtype != torch.float32:
            raise ValueError("S_prefix/Z_prefix must be float32")
        if Z_prefix.shape[0] != n_prefix:
            raise ValueError("S_prefix and Z_prefix hold different segment counts")
    if out is None:
        out = torch.empty_like(q_seg)
    _dev(out)
    _check(lib.rehyat_segment_attend(d, _dtype_code(q_seg), T, frame_tokens, Tc, To, c0, c1,
                                     _ptr(q_seg), _ptr(k_seg), _ptr(v_seg), _ptr(Wq), _ptr(bq),
                                     n_prefix, _ptr(S_prefix), _ptr(Z_prefix), _ptr(out),
                                     _ptr(workspace), workspace.numel(), _stream(dev)))
    return out


def forward_states(k, v, Wk, bk, *, P: int, phi: int = 0, frame_tokens: int, Tc: int, To: int,
                   workspace: torch.Tensor) -> torch.Tensor:
    """First phase of `forward`: fills `workspace` with the state every chunk reads."""
    lib = load()
    _check_x_w(k, Wk, bk, "k")
    _shape(v, k.shape, "v")
    _frames(k.shape[2], frame_tokens, "k")
    dev = _dev(k, v, Wk, bk, workspace)
    d = dims_of(k, Wk, P, phi)
    T = k.shape[2] // frame_tokens
    _check(lib.rehyat_forward_states(d, _dtype_code(k), T, frame_tokens, Tc, To, _ptr(k), _ptr(v),
                                     _ptr(Wk), _ptr(bk), _ptr(workspace), workspace.numel(),
                                     _stream(dev)))
    return workspace


def forward_phiq(q, Wq, bq, *, P: int, phi: int = 0, frame_tokens: int, Tc: int, To: int,
                 workspace: torch.Tensor) -> torch.Tensor:
    """Second phase of `forward`: phi_q of the query rows that read a state, into `workspace`."""
    lib = load()
    _check_x_w(q, Wq, bq, "q")
    _frames(q.shape[2], frame_tokens, "q")
    dev = _dev(q, Wq, bq, workspace)
    d = dims_of(q, Wq, P, phi)
    T = q.shape[2] // frame_tokens
    _check(lib.rehyat_forward_phiq(d, _dtype_code(q), T, frame_tokens, Tc, To, _ptr(q), _ptr(Wq),
                                   _ptr(bq), _ptr(workspace), workspace.numel(), _stream(dev)))
    return workspace


def forward_attend(q, k, v, *, dims: Dims, frame_tokens: int, Tc: int, To: int,
                   workspace: torch.Tensor, out: torch.Tensor) -> torch.Tensor:
    """Third phase of `forward`: the hybrid output from q, k, v and the workspace."""
    lib = load()
    for t, n in ((k, "k"), (v, "v"), (out, "out")):
        _shape(t, q.shape, n)
    _frames(q.shape[2], frame_tokens, "q")
    dev = _dev(q, k, v, workspace, out)
    T = q.shape[2] // frame_tokens
    _check(lib.rehyat_forward_attend(dims, _dtype_code(q), T, frame_tokens, Tc, To, _ptr(q),
                                     _ptr(k), _ptr(v), _ptr(out), _ptr(workspace),
                                     workspace.numel(), _stream(dev)))
    return out


def chunk_states(k, v, Wk, bk, *, P: int, phi: int = 0, frame_tokens: int, Tc: int, To: int,
                 workspace: torch.Tensor | None = None):
    """States each chunk of `forward` reads: S [B,H,C,F,D], Z [B,H,C,F] (fp32)."""
    lib = load()
    _check_x_w(k, Wk, bk, "k")
    _shape(v, k.shape, "v")
    _frames(k.shape[2], frame_tokens, "k")
    dev = _dev(k, v, Wk, bk)
    d = dims_of(k, Wk, P, phi)
    N = k.shape[2]
    T = N // frame_tokens
    C = -(-T // Tc)
    code = _dtype_code(k)
    ws = _workspace(forward_workspace_size(d, code, T, frame_tokens, Tc, To), dev, workspace)
    S = torch.empty(d.B, d.H, C, d.F, d.D, dtype=torch.float32, device=dev)
    Z = torch.empty(d.B, d.H, C, d.F, dtype=torch.float32, device=dev)
    _check(lib.rehyat_chunk_states(d, code, T, frame_tokens, Tc, To, _ptr(k), _ptr(v), _ptr(Wk),
                                   _ptr(bk), _ptr(S), _ptr(Z), _ptr(ws), ws.numel(),
                                   _stream(dev)))
    return S, Z


def chunk_forward(q, k_win, v_win, Wq, bq, Wk, bk, S, Z, *, P: int, phi: int = 0, frame_tokens: int,
                  frames_before: int, To: int, To_next: int | None = None,
                  out: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """One streaming step; S [B,H,F,D] and Z [B,H,F] (fp32) are updated in place.  To_next (the
    overlap of the next call, for a variable schedule) defaults to To."""
    lib = load()
    cf = _frames(q.shape[2], frame_tokens, "q")
    _check_step(q, k_win, v_win, Wq, bq, Wk, bk, S, Z, out, frame_tokens,
                min(To, frames_before) + cf, "k_win")
    dev = _dev(q, k_win, v_win, Wq, bq, Wk, bk, S, Z)
    d = dims_of(q, Wq, P, phi)
    chunk_frames = q.shape[2] // frame_tokens
    code = _dtype_code(q)
    ws = _workspace(chunk_workspace_size(d, code, frame_tokens, chunk_frames, To), dev, workspace)
    if out is None:
        out = torch.empty_like(q)
    args = (_ptr(q), _ptr(k_win), _ptr(v_win), _ptr(Wq), _ptr(bq), _ptr(Wk), _ptr(bk), _ptr(S),
            _ptr(Z), _ptr(out), _ptr(ws), ws.numel(), _stream(dev))
    if To_next is None:
        _check(lib.rehyat_chunk_forward(d, code, frame_tokens, frames_before, chunk_frames, To,
                                        *args))
    else:
        _check(lib.rehyat_chunk_forward_sched(d, code, frame_tokens, frames_before, chunk_frames,
                                              To, To_next, *args))
    return out


def chunk_carry_workspace_size(d: Dims, dtype_code: int, L_: int, chunk_frames: int, To: int,
                               carry_frames: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().rehyat_chunk_carry_workspace_size(d, dtype_code, L_, chunk_frames, To,
                                                    carry_frames, ctypes.byref(n)))
    return n.value


def chunk_forward_carry(q, k, v, Wq, bq, Wk, bk, S, Z, k_carry, v_carry, *, P: int, phi: int = 0,
                        frame_tokens: int, frames_before: int, To: int,
                        To_next: int | None = None, out: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None):
    """Streaming step on the chunk alone; S, Z and the carried frames k_carry, v_carry
    [B,H,carry_frames*L,D] are updated in place."""
    lib = load()
    _check_step(q, k, v, Wq, bq, Wk, bk, S, Z, out, frame_tokens, None, "k")
    _frames(k_carry.shape[2], frame_tokens, "k_carry")
    _shape(k_carry, (q.shape[0], q.shape[1], k_carry.shape[2], q.shape[3]), "k_carry")
    _shape(v_carry, k_carry.shape, "v_carry")
    dev = _dev(q, k, v, Wq, bq, Wk, bk, S, Z, k_carry, v_carry)
    d = dims_of(q, Wq, P, phi)
    chunk_frames = q.shape[2] // frame_tokens
    carry_frames = k_carry.shape[2] // frame_tokens
    code = _dtype_code(q)
    ws = _workspace(chunk_carry_workspace_size(d, code, frame_tokens, chunk_frames, To,
                                               carry_frames), dev, workspace)
    if out is None:
        out = torch.empty_like(q)
    _check(lib.rehyat_chunk_forward_carry(d, code, frame_tokens, frames_before, chunk_frames, To,
                                          To if To_next is None else To_next, carry_frames,
                                          _ptr(q), _ptr(k), _ptr(v), _ptr(Wq), _ptr(bq),
                                          _ptr(Wk), _ptr(bk), _ptr(S), _ptr(Z), _ptr(k_carry),
                                          _ptr(v_carry), _ptr(out), _ptr(ws), ws.numel(),
                                          _stream(dev)))
    return out


def chunk_forward_static(q, k_win, v_win, Wq, bq, Wk, bk, S, Z, *, P: int, phi: int = 0, frame_tokens: int,
                         frames_before: int, To: int, out: torch.Tensor | None = None):
    """chunk_forward without a workspace: the library's own fixed device scratch is used (for
    callers that cannot allocate); bf16 only."""
    lib = load()
    cf = _frames(q.shape[2], frame_tokens, "q")
    _check_step(q, k_win, v_win, Wq, bq, Wk, bk, S, Z, out, frame_tokens,
                min(To, frames_before) + cf, "k_win")
    dev = _dev(q, k_win, v_win, Wq, bq, Wk, bk, S, Z)
    d = dims_of(q, Wq, P, phi)
    chunk_frames = q.shape[2] // frame_tokens
    if out is None:
        out = torch.empty_like(q)
    _check(lib.rehyat_chunk_forward_static(d, _dtype_code(q), frame_tokens, frames_before,
                                           chunk_frames, To, _ptr(q), _ptr(k_win), _ptr(v_win),
                                           _ptr(Wq), _ptr(bq), _ptr(Wk), _ptr(bk), _ptr(S),
                                           _ptr(Z), _ptr(out), _stream(dev)))
    return out


def forward_train(q, k, v, Wq, bq, Wk, bk, *, P: int, phi: int = 0, frame_tokens: int, Tc: int,
                  To: int, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """`forward` that also returns lse [B,H,N] fp32 (log2 of every row's denominator), which
    `backward` needs.  bf16 only."""
    lib = load()
    _check_x_w(q, Wq, bq, "q")
    _check_x_w(q, Wk, bk, "q")
    _shape(Wk, Wq.shape, "Wk")
    for t, n in ((k, "k"), (v, "v"), (out, "out")):
        _shape(t, q.shape, n)
    _frames(q.shape[2], frame_tokens, "q")
    dev = _dev(q, k, v, Wq, bq, Wk, bk)
    _weights(Wq, bq), _weights(Wk, bk)
    d = dims_of(q, Wq, P, phi)
    N = q.shape[2]
    T = N // frame_tokens
    code = _dtype_code(q)
    ws = _workspace(forward_workspace_size(d, code, T, frame_tokens, Tc, To), dev, workspace)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], N, dtype=torch.float32, device=dev)
    _check(lib.rehyat_forward_train(d, code, T, frame_tokens, Tc, To, _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(Wq), _ptr(bq), _ptr(Wk), _ptr(bk), _ptr(out), _ptr(lse),
                                    _ptr(ws), ws.numel(), _stream(dev)))
    return out, lse


def backward_workspace_size(d: Dims, dtype_code: int, T: int, L_: int, Tc: int, To: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().rehyat_backward_workspace_size(d, dtype_code, T, L_, Tc, To, ctypes.byref(n)))
    return n.value


GRAD_NAMES = ("dq", "dk", "dv", "dWq", "dbq", "dWk", "dbk")


def backward(q, k, v, Wq, bq, Wk, bk, out, lse, dout, *, P: int, phi: int = 0,
             frame_tokens: int, Tc: int, To: int, workspace: torch.Tensor | None = None,
             grads: dict | None = None) -> dict:
    """Gradients of sum(dout * out) for every input: dict with dq, dk, dv [B,H,N,D], dWq, dWk
    [H,G,F/G,D/G], dbq, dbk [H,F] (fp32).  `grads` may hold those buffers (written, not added
    to)."""
    lib = load()
    _check_x_w(q, Wq, bq, "q")
    _check_x_w(q, Wk, bk, "q")
    _shape(Wk, Wq.shape, "Wk")
    for t, n in ((k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _shape(t, q.shape, n)
    _shape(lse, q.shape[:3], "lse")
    _frames(q.shape[2], frame_tokens, "q")
    dev = _dev(q, k, v, Wq, bq, Wk, bk, out, lse, dout)
    d = dims_of(q, Wq, P, phi)
    N = q.shape[2]
    T = N // frame_tokens
    code = _dtype_code(q)
    ws = _workspace(backward_workspace_size(d, code, T, frame_tokens, Tc, To), dev, workspace)
    shapes = {"dq": q.shape, "dk": q.shape, "dv": q.shape, "dWq": Wq.shape, "dWk": Wk.shape,
              "dbq": (d.H, d.F), "dbk": (d.H, d.F)}
    g = {}
    for n in GRAD_NAMES:
        t = grads.get(n) if grads is not None else None
        if t is None:
            t = torch.empty(shapes[n], dtype=torch.float32, device=dev)
        elif tuple(t.shape) != tuple(shapes[n]) or t.dtype != torch.float32:
            raise ValueError(f"grads[{n!r}] must be float32 of shape {tuple(shapes[n])}")
        g[n] = t
    _dev(*g.values())
    _check(lib.rehyat_backward(d, code, T, frame_tokens, Tc, To, _ptr(q), _ptr(k), _ptr(v),
                               _ptr(Wq), _ptr(bq), _ptr(Wk), _ptr(bk), _ptr(out), _ptr(lse),
                               _ptr(dout), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                               _ptr(g["dWq"]), _ptr(g["dbq"]), _ptr(g["dWk"]), _ptr(g["dbk"]),
                               _ptr(ws), ws.numel(), _stream(dev)))
    return g


def gemm(A: torch.Tensor, B: torch.Tensor, *, a_mn: bool = False, b_mn: bool = False,
         out: torch.Tensor | None = None, accumulate: bool = False, alpha: float = 1.0,
         out_dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """Batched bf16 GEMM on the tensor cores.  A [batch, M, K] (or [batch, K, M] with a_mn),
    B [batch, N, K] (or [batch, K, N] with b_mn), both contiguous bf16; returns C [batch, M, N]
    = alpha A B (added to `out` with accumulate)."""
    dev = _dev(A, B)
    batch = A.shape[0]
    M, K = (A.shape[2], A.shape[1]) if a_mn else (A.shape[1], A.shape[2])
    N = B.shape[2] if b_mn else B.shape[1]
    if out is None:
        out = torch.empty(batch, M, N, dtype=out_dtype, device=dev)
    _check(load().rehyat_gemm_bf16(M, N, K, batch, _ptr(A), A.shape[2], A.shape[1] * A.shape[2],
                                   int(a_mn), _ptr(B), B.shape[2], B.shape[1] * B.shape[2],
                                   int(b_mn), _ptr(out), out.shape[2], out.shape[1] * out.shape[2],
                                   int(out.dtype == torch.bfloat16), int(accumulate),
                                   ctypes.c_float(alpha), _stream(dev)))
    return out


def selftest_bounds(buf: torch.Tensor, n: int, bad_index: int) -> None:
    """Enqueue the debug-bounds self test on buf (fp32, at least n + 1 elements past which
    bad_index must stay)."""
    if buf.dtype != torch.float32 or buf.numel() <= max(n, bad_index):
        raise ValueError("buf must be fp32 with room for index max(n, bad_index)")
    dev = _dev(buf)
    _check(load().rehyat_selftest_bounds(_ptr(buf), n, bad_index, _stream(dev)))


def selftest_wait_timeout(limit_ns: int = 20_000_000, device: torch.device | None = None) -> None:
    """Enqueue the bounded-wait failure self test; the next sync_status() then raises
    RehyatError with status REHYAT_ERR_TIMEOUT."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    _check(load().rehyat_selftest_wait_timeout(ctypes.c_longlong(int(limit_ns)), _stream(dev)))


def sync_status(device: torch.device | None = None) -> None:
    """Synchronise the current stream and raise if a kernel reported a device-side failure."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    _check(load().rehyat_sync_status(_stream(dev)))
