"""Fits the polynomial the kernels use for log1p(w) on [0, 1].

    log1p(w) ~= w * P(w),   P of degree 9,

chosen to minimise the maximum relative error over [0, 1] (Lawson's iteratively reweighted
least squares on a dense Chebyshev grid, which converges to the minimax fit).  Run it to
reproduce the coefficients in csrc/device_math.cuh:

    python -m selective_state_space_silu_b200.fit_log1p
"""

import numpy as np

DEGREE = 9


def fit(degree: int = DEGREE, iters: int = 400):
    k = np.arange(20001)
    w = 0.5 - 0.5 * np.cos(np.pi * k / k[-1])           # Chebyshev-spaced on [0, 1]
    w = w[1:]                                           # P(0) = 1 is implied by the fit
    target = np.log1p(w) / w                            # P(w); relative error of w*P = of P
    V = np.vander(w, degree + 1, increasing=True)
    wt = np.ones_like(w)
    for _ in range(iters):
        A = V * (wt / target)[:, None]
        c, *_ = np.linalg.lstsq(A, wt, rcond=None)
        err = np.abs(V @ c / target - 1.0)
        wt = wt * (err + 1e-30) ** 0.5
        wt /= wt.sum()
    return c


def max_rel_err_f32(c):
    w = np.linspace(0.0, 1.0, 2_000_001, dtype=np.float32)[1:]
    cf = c.astype(np.float32)
    p = np.full_like(w, cf[-1])
    for a in cf[-2::-1]:
        p = (p * w + a).astype(np.float32)
    got = (w * p).astype(np.float64)
    ref = np.log1p(w.astype(np.float64))
    return float(np.max(np.abs(got / ref - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, a in enumerate(c):
        print(f"c{i} = {np.float32(a)!r}")
    print("max relative error (fp32 Horner):", max_rel_err_f32(c))
