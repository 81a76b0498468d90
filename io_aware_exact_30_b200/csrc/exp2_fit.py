"""Coefficients of the polynomial exp2 used by the kernels (``exp2_poly`` in
ptx.cuh), and the check of their error bound.

Method: Cody-Waite style range reduction x = j + f with j = round(x) and
f in [-1/2, 1/2] (W. J. Cody and W. Waite, "Software Manual for the
Elementary Functions", 1980), so 2^x = 2^j * 2^f; 2^f is a degree-3
polynomial with p(0) = 1 whose other coefficients minimise the maximum
relative error on [-1/2, 1/2] (iteratively re-weighted least squares on
Chebyshev nodes, converging to the equi-oscillating solution); 2^j is added
to the exponent field.  The kernels evaluate a fraction of each row's
exponentials this way on the FMA pipe and the rest with ex2.approx on the
multi-function unit, which would otherwise bound the softmax.

    python io_aware_exact_30_b200/csrc/exp2_fit.py   # prints the coefficients
"""

import numpy as np

DEGREE = 3
# The values written into ptx.cuh (fp32, printed by fit()).
COEFFS = (0.693282961845398, 0.2422109991312027, 0.0550089068710804)
MAX_REL_ERR = 1.02e-4


def fit(degree: int = DEGREE):
    f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5
    w = np.ones_like(f)
    for _ in range(60):
        A = np.stack([f ** k for k in range(1, degree + 1)], 1) / (2 ** f)[:, None]
        b = (2 ** f - 1) / 2 ** f
        W = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * W[:, None], b * W, rcond=None)
        p = 1 + sum(c[k - 1] * f ** k for k in range(1, degree + 1))
        err = np.abs(p / 2 ** f - 1)
        w = w * (1 + 10 * err / err.max())
    return tuple(float(x) for x in np.float32(c)), float(err.max())


def emulate(x):
    """fp32 emulation of the device routine (same operation order)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23: t's low mantissa bits hold round(x)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    c1, c2, c3 = (np.float32(c) for c in COEFFS)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


if __name__ == "__main__":
    c, e = fit()
    print("coefficients", c, "max relative error", e)
