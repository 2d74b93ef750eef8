"""The feature-map kernels' softplus (featmap.cuh: softplus_log2_x2 and phi16's single-power
path), emulated step by step in fp32 on the CPU with the constants read from the header, against
softplus(u)^p in float64.  Also checks that the header's constants are the fit script's output,
and that the error bound would catch a wrong coefficient."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "hybrid_softmax_linear_chunked_b200", "csrc")
HEADER = os.path.join(CSRC, "featmap.cuh")
# fp32 emulation error budget: quintic 8.6e-6, rounding of t = u log2(e) (relative error of
# 2^-|t| about |t| * 2^-24 * ln 2, below 6e-6 for |t| <= 116) and a few fp32 roundings per step,
# times p for the power; far below the 2^-9 relative rounding of the bf16 result.
BOUND = 5e-5


def header_constants():
    text = open(HEADER).read()
    out = {}
    for name in ("kL1pC0", "kL1pC1", "kL1pC2", "kL1pC3", "kL1pC4", "kL1pC5", "kLog2e", "kLn2"):
        m = re.search(rf"constexpr float {name} = ([-+0-9.eE]+)f;", text)
        assert m, name
        out[name] = np.float32(float(m.group(1)))
    return out


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fma32(a, b, c):
    # one rounding, as fma.rn.f32 (the float64 product of two fp32 values is exact)
    return f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def device_phi(u, bias, p, scale, k):
    """phi16's single-power path for one feature, in the kernel's order of fp32 operations."""
    c = [k[f"kL1pC{i}"] for i in range(6)]
    x = f32(f32(u).astype(np.float64) + np.float64(np.float32(bias)))
    t = f32(x.astype(np.float64) * np.float64(k["kLog2e"]))
    y = f32(np.exp2(-np.abs(t.astype(np.float64))))
    y = np.where(y < np.float32(2.0 ** -126), np.float32(0.0), y)  # ex2.approx.ftz
    r = fma32(np.full_like(y, c[5]), y, np.full_like(y, c[4]))
    for ci in (c[3], c[2], c[1], c[0]):
        r = fma32(r, y, np.full_like(y, ci))
    s = fma32(r, y, np.maximum(t, np.float32(0.0)))
    ln2 = k["kLn2"]
    fac = {1: f32(ln2 * np.float32(scale)),
           2: f32(f32(ln2 * ln2) * np.float32(scale)),
           3: f32(f32(f32(ln2 * ln2) * ln2) * np.float32(scale))}[p]
    v = s
    if p == 2:
        v = f32(s.astype(np.float64) * s)
    if p == 3:
        v = f32(f32(s.astype(np.float64) * s).astype(np.float64) * s)
    return f32(v.astype(np.float64) * np.float64(fac))


def softplus64(x):
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


U = np.concatenate([np.linspace(-80.0, 40.0, 120001), np.linspace(-1e-3, 1e-3, 2001)])


@pytest.mark.parametrize("p", [1, 2, 3])
@pytest.mark.parametrize("bias,scale", [(0.0, 1.0), (0.37, 1.0), (-1.25, 0.015625)])
def test_device_softplus_power_within_bound(p, bias, scale):
    k = header_constants()
    # u >= -80 / p keeps softplus(u)^p inside the normal fp32 range (e^-80 is about 2^-115)
    u = U[U >= -80.0 / p]
    got = device_phi(u, bias, p, scale, k).astype(np.float64)
    x = f32(f32(u).astype(np.float64) + np.float64(np.float32(bias))).astype(np.float64)
    want = softplus64(x) ** p * np.float64(np.float32(scale))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= BOUND, f"max relative error {rel.max():.3e} at u = {u[rel.argmax()]}"


def test_bound_catches_a_wrong_coefficient():
    k = header_constants()
    k["kL1pC3"] = np.float32(k["kL1pC3"] * 1.01)
    got = device_phi(U, 0.0, 1, 1.0, k).astype(np.float64)
    want = softplus64(f32(U).astype(np.float64))
    assert np.abs(got / want - 1.0).max() > BOUND


def test_header_constants_are_the_fit():
    spec = importlib.util.spec_from_file_location("softplus_poly_fit",
                                                  os.path.join(CSRC, "softplus_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    coef = mod.fit()
    k = header_constants()
    for i, cval in enumerate(coef):
        assert k[f"kL1pC{i}"] == np.float32(cval), i
    assert k["kLog2e"] == np.float32(1.0 / np.log(2.0))
    assert k["kLn2"] == np.float32(np.log(2.0))
