"""Host-side checks of librehyat.so that need no GPU: it loads, exports every function the header
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from hybrid_softmax_linear_chunked_b200 import binding as rb
from hybrid_softmax_linear_chunked_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "rehyat.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return rb.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rehyat_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_surface():
    assert declared_functions() == sorted(rb.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.rehyat_version() == 102


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced: checks come first


def dims(B=1, H=2, D=128, F=128, G=8, P=2, phi=0):
    return rb.Dims(B, H, D, F, G, P, phi)


def call_forward(lib, d, dt=rb.REHYAT_BF16, T=7, L=64, Tc=3, To=1, ws_bytes=1 << 40, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, Wq=FAKE, bq=None, Wk=FAKE, bk=None, out=FAKE, ws=FAKE)
    p.update(ptrs)
    return lib.rehyat_forward(d, dt, T, L, Tc, To, p["q"], p["k"], p["v"], p["Wq"], p["bq"],
                              p["Wk"], p["bk"], p["out"], p["ws"], ws_bytes, None)


@pytest.mark.parametrize("kwargs,status", [
    (dict(d=dims(B=0)), -1),
    (dict(d=dims(G=3)), -1),
    (dict(d=dims(P=200)), -1),
    (dict(d=dims(phi=2)), -1),
    (dict(d=dims(phi=-1)), -1),
    (dict(d=dims(D=64, F=64)), -2),
    (dict(d=dims(F=64)), -2),
    (dict(d=dims(), dt=7), -3),
    (dict(d=dims(), Tc=0), -1),
    (dict(d=dims(), To=-1), -1),
    (dict(d=dims(), T=0), -1),
    (dict(d=dims(), ws_bytes=16), -4),
    (dict(d=dims(), q=None), -1),
    (dict(d=dims(), q=ctypes.c_void_p(0x10008)), -7),
    (dict(d=dims(D=48, F=48, G=4), dt=rb.REHYAT_F32), -2),
])
def test_forward_rejects_bad_arguments(lib, kwargs, status):
    assert call_forward(lib, **kwargs) == status
    assert lib.rehyat_last_error().decode()


def test_workspace_sizes(lib):
    n = ctypes.c_size_t(0)
    assert lib.rehyat_forward_workspace_size(dims(H=12), rb.REHYAT_BF16, 21, 1560, 3, 1,
                                             ctypes.byref(n)) == 0
    # 6 folds x splits x (F*D + F) fp32 partials, 7 transposed bf16 states, 7 Z vectors
    assert n.value >= 12 * (7 * 128 * 128 * 2 + 7 * 128 * 4)
    m = ctypes.c_size_t(0)
    assert lib.rehyat_chunk_workspace_size(dims(B=2, H=12), rb.REHYAT_BF16, 1560, 3, 1,
                                           ctypes.byref(m)) == 0
    # streaming workspace does not depend on how long the video is
    assert m.value < 64 << 20


def test_chunk_forward_rejects_bad_arguments(lib):
    d = dims()
    st = lib.rehyat_chunk_forward(d, rb.REHYAT_BF16, 64, -1, 3, 1, FAKE, FAKE, FAKE, FAKE, None,
                                  FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == -1
    st = lib.rehyat_chunk_forward(d, rb.REHYAT_BF16, 64, 3, 3, 1, FAKE, FAKE, FAKE, FAKE, None,
                                  FAKE, None, None, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == -1
    st = lib.rehyat_chunk_forward(d, rb.REHYAT_BF16, 64, 3, 3, 1, FAKE, FAKE, FAKE, FAKE, None,
                                  FAKE, None, FAKE, FAKE, FAKE, FAKE, 8, None)
    assert st == -4


def test_selftest_rejects_limits_out_of_range(lib):
    for bad in (0, 999, 2_000_000_001):
        assert lib.rehyat_selftest_wait_timeout(bad, None) == -1
        assert "limit_ns" in lib.rehyat_last_error().decode()


def test_abi_version_and_dims_layout(lib):
    assert lib.rehyat_version() == 102
    assert ctypes.sizeof(rb.Dims) == 7 * 4
    # the elu + 1 kind passes validation (workspace queries need no device)
    n = ctypes.c_size_t(0)
    assert lib.rehyat_forward_workspace_size(dims(phi=rb.PHI_ELU1), rb.REHYAT_BF16, 7, 64, 3, 1,
                                             ctypes.byref(n)) == 0 and n.value > 0


def test_chunk_forward_sched_rejects_overlap_into_folded_frames(lib):
    d = dims()
    # window of frames [2, 4) (To = 1 after 3 frames, 1-frame chunk): a next overlap of 3 would
    # need frame 1, already folded into S
    st = lib.rehyat_chunk_forward_sched(d, rb.REHYAT_BF16, 64, 3, 1, 1, 3, FAKE, FAKE, FAKE, FAKE,
                                        None, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == -1 and "folded" in lib.rehyat_last_error().decode()
    st = lib.rehyat_chunk_forward_sched(d, rb.REHYAT_BF16, 64, 3, 1, 1, -1, FAKE, FAKE, FAKE, FAKE,
                                        None, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == -1


def test_chunk_forward_carry_checks(lib):
    d = dims()
    n = ctypes.c_size_t(0)
    assert lib.rehyat_chunk_carry_workspace_size(d, rb.REHYAT_BF16, 64, 3, 2, 1, ctypes.byref(n)) == -1
    assert lib.rehyat_chunk_carry_workspace_size(d, rb.REHYAT_BF16, 64, 3, 1, 1, ctypes.byref(n)) == 0
    # carry shorter than the overlap
    st = lib.rehyat_chunk_forward_carry(d, rb.REHYAT_BF16, 64, 3, 3, 2, 2, 1, FAKE, FAKE, FAKE,
                                        FAKE, None, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, 1 << 30, None)
    assert st == -1 and "carry_frames" in lib.rehyat_last_error().decode()
    # workspace too small
    st = lib.rehyat_chunk_forward_carry(d, rb.REHYAT_BF16, 64, 3, 3, 1, 1, 1, FAKE, FAKE, FAKE,
                                        FAKE, None, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, 16, None)
    assert st == -4


def test_backward_checks(lib):
    d = dims()
    n = ctypes.c_size_t(0)
    assert lib.rehyat_backward_workspace_size(d, rb.REHYAT_F32, 7, 64, 3, 1, ctypes.byref(n)) == -3
    assert lib.rehyat_backward_workspace_size(d, rb.REHYAT_BF16, 7, 64, 3, 1, ctypes.byref(n)) == 0
    args = [FAKE] * 3 + [FAKE, None, FAKE, None] + [FAKE] * 3 + [FAKE] * 7 + [FAKE]
    # frame_tokens not a multiple of 8
    assert lib.rehyat_backward(d, rb.REHYAT_BF16, 7, 60, 3, 1, *args, 1 << 40, None) == -2
    # workspace too small
    assert lib.rehyat_backward(d, rb.REHYAT_BF16, 7, 64, 3, 1, *args, 16, None) == -4
    # fp32 training forward refused
    assert lib.rehyat_forward_train(d, rb.REHYAT_F32, 7, 64, 3, 1, FAKE, FAKE, FAKE, FAKE, None,
                                    FAKE, None, FAKE, FAKE, FAKE, 1 << 40, None) == -3


def test_segment_checks(lib):
    """Context-parallel segment calls: range, dtype and workspace checks (no device work)."""
    d = dims()
    n = ctypes.c_size_t(0)
    # 7 chunks of 3 frames (T = 21): [2, 5) is a valid segment
    assert lib.rehyat_segment_workspace_size(d, rb.REHYAT_BF16, 21, 64, 3, 1, 2, 5,
                                             ctypes.byref(n)) == 0 and n.value > 0
    for c0, c1 in [(3, 3), (-1, 2), (5, 8)]:
        assert lib.rehyat_segment_workspace_size(d, rb.REHYAT_BF16, 21, 64, 3, 1, c0, c1,
                                                 ctypes.byref(n)) == -1
    assert lib.rehyat_segment_workspace_size(d, rb.REHYAT_F32, 21, 64, 3, 1, 0, 7,
                                             ctypes.byref(n)) == -3
    # the segment sums need a workspace at least the plan's size
    st = lib.rehyat_segment_states(d, rb.REHYAT_BF16, 21, 64, 3, 1, 2, 5, FAKE, FAKE, FAKE, None,
                                   FAKE, FAKE, FAKE, 16, None)
    assert st == -4
    # prefix states announced but missing
    st = lib.rehyat_segment_attend(d, rb.REHYAT_BF16, 21, 64, 3, 1, 2, 5, FAKE, FAKE, FAKE, FAKE,
                                   None, 2, None, None, FAKE, FAKE, 1 << 30, None)
    assert st == -1 and "S_prefix" in lib.rehyat_last_error().decode()


def test_static_chunk_refuses_problems_beyond_its_scratch(lib):
    """The static-scratch streaming call needs B*H*(6FD + 4F) + 4HFD bytes with one fold split;
    past 16 MiB it refuses before anything is enqueued (no device is touched here)."""
    def call(B, H):
        return lib.rehyat_chunk_forward_static(dims(B=B, H=H), rb.REHYAT_BF16, 64, 3, 3, 1, FAKE,
                                               FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE,
                                               FAKE, None)
    for B, H in [(14, 12), (1, 200), (170, 1)]:
        assert call(B, H) == -4, (B, H)
        assert "scratch" in lib.rehyat_last_error().decode()


def test_release_build_has_no_bounds_checks(lib):
    """The default library is built without the debug-bounds checks; its self test says so
    instead of launching anything."""
    assert lib.rehyat_debug_bounds() == 0
    assert lib.rehyat_selftest_bounds(FAKE, 16, 20, None) == -1
    assert "debug-bounds" in lib.rehyat_last_error().decode()
