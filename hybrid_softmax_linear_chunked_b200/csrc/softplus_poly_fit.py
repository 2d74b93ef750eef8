"""Fits the quintic r(y) ~ log2(1 + y) / y on [0, 1] used by the feature-map kernels
(featmap.cuh, kL1pC0..kL1pC5) for softplus in log2 units: log2(1 + y) = y r(y) with
y = 2^-|t|.  The fit minimises the maximum relative error by iteratively reweighted least
squares (Lawson's algorithm) on a dense grid; the printed constants are rounded to fp32.

    python softplus_poly_fit.py        # prints the coefficients and the error of the fp32 form
"""
import numpy as np

DEGREE = 5


def ratio(y: np.ndarray) -> np.ndarray:
    """log2(1 + y) / y, continued by its limit 1/ln 2 at y = 0."""
    out = np.empty_like(y)
    small = y < 1e-8
    out[~small] = np.log2(1.0 + y[~small]) / y[~small]
    out[small] = (1.0 - y[small] / 2.0) / np.log(2.0)
    return out


def fit(degree: int = DEGREE, iters: int = 300, n_grid: int = 40001) -> np.ndarray:
    """Coefficients c[0..degree] (increasing powers) minimising max |p(y) / r(y) - 1| on [0, 1]."""
    y = np.linspace(0.0, 1.0, n_grid)
    target = ratio(y)
    A = np.vander(y, degree + 1, increasing=True) / target[:, None]
    w = np.full_like(y, 1.0 / n_grid)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        err = np.abs(A @ c - 1.0)
        w = w * (err + 1e-30)
        w /= w.sum()
    return c


def fp32_log2_1p(c: np.ndarray, y: np.ndarray) -> np.ndarray:
    """y r(y) in the kernels' order: Horner in fp32 with fused multiply-adds, the last one
    multiplying by y."""
    c32 = np.asarray(c, dtype=np.float32)
    y32 = y.astype(np.float32)
    r = c32[-1]
    for k in range(len(c32) - 2, -1, -1):
        r = (r.astype(np.float64) * y32 + c32[k]).astype(np.float32)
    return (r.astype(np.float64) * y32).astype(np.float32)


if __name__ == "__main__":
    coef = fit()
    y = np.linspace(0.0, 1.0, 100001)[1:]
    rel = np.abs(fp32_log2_1p(coef, y).astype(np.float64) / np.log2(1.0 + y) - 1.0).max()
    for k, v in enumerate(coef):
        print(f"kL1pC{k} = {np.float32(v)!r}")
    print(f"max relative error of y r(y) in fp32: {rel:.2e}")
