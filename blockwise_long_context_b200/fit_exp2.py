"""Fits the cubic that approximates 2^f on [-1/2, 1/2] for the forward kernel.

The softmax exponentials are split between the special-function unit
(ex2.approx) and the FMA pipe.  On the FMA pipe, 2^x is evaluated by
rounding x to the nearest integer n (x = n + f, |f| <= 1/2), evaluating
p(f) ~ 2^f with the cubic fitted here, and adding n to the exponent field.
The cubic minimises the maximum relative error over [-1/2, 1/2] by
iteratively reweighted least squares on Chebyshev nodes.

    python -m blockwise_long_context_b200.fit_exp2

prints the fp32 coefficients (c0, c1, c2, c3) and the maximum relative
error of the fp32 Horner evaluation; the values are embedded in
csrc/lvx_ptx.cuh and a CPU test re-runs this fit to check them.
"""

import numpy as np


def fit(iterations: int = 60):
    f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5
    y = np.exp2(f)
    w = 1 / y
    V = np.vander(f, 4, increasing=True)
    for _ in range(iterations):
        c, *_ = np.linalg.lstsq(V * w[:, None], y * w, rcond=None)
        err = (V @ c - y) / y
        w = w * (1 + 2 * np.abs(err) / np.abs(err).max())
        w /= w.mean()
    return c.astype(np.float32)


def max_rel_error(c32) -> float:
    ff = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = ((c32[3] * ff + c32[2]) * ff + c32[1]) * ff + c32[0]
    return float(np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1).max())


if __name__ == "__main__":
    c = fit()
    print("coefficients:", ", ".join(f"{float(x):.9e}f" for x in c))
    print("max relative error:", max_rel_error(c))
