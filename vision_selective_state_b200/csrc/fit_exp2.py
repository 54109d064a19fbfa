"""Least-squares fit of q(f) ~ (2^f - 1) / f on f in [-1/2, 1/2] (Chebyshev nodes).

The scan kernels can evaluate part of their retentions 2^x on the FMA pipe
instead of the special-function unit. The range reduction is the classic one
(Cody and Waite, "Software Manual for the Elementary Functions", 1980): with
k = round(x) and f = x - k in [-1/2, 1/2],

    2^x = 2^k * 2^f,   2^f = 1 + f * q(f),

and 2^k is added to the exponent field of the result. Writing 2^f as
1 + f * q(f) makes 2^0 exactly 1 (a zero step keeps the state unchanged, as the
SFU's ex2 does). The fit weights the residual by f / 2^f so that it minimises
the relative error of 2^f. Run to regenerate the coefficients in
vscan_common.cuh and to print the relative error of the fp64 fit and of a
float32 Horner evaluation.
"""
import numpy as np


def fit(degree, nodes=4000):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    f = f[np.abs(f) > 1e-12]
    target = np.expm1(f * np.log(2.0)) / f          # (2^f - 1) / f
    w = np.abs(f) / np.exp2(f)                       # residual of q -> relative residual of 2^f
    V = np.vander(f, degree + 1, increasing=True)
    c, *_ = np.linalg.lstsq(V * w[:, None], target * w, rcond=None)
    return c


def rel_err(c, fp32=False):
    f = np.linspace(-0.5, 0.5, 400001)
    if fp32:
        f32 = f.astype(np.float32)
        acc = np.float32(c[-1])
        for ci in c[-2::-1]:
            acc = (acc * f32 + np.float32(ci)).astype(np.float32)
        p = (np.float32(1.0) + f32 * acc).astype(np.float64)
        f = f32.astype(np.float64)
    else:
        p = 1.0 + f * np.polyval(c[::-1], f)
    exact = np.exp2(f)
    return float(np.max(np.abs(p - exact) / exact))


if __name__ == "__main__":
    for d in range(3, 8):
        c = fit(d)
        print(f"q degree {d}: rel err {rel_err(c):.2e} (fp64)  {rel_err(c, True):.2e} (fp32 Horner)")
    c = fit(5)
    print("coefficients of q, degree 5, c0..c5:")
    for ci in c:
        print(f"    {float(np.float32(ci)):.9e}f,")
