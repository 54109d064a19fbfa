"""Least-squares fit of Q(x) ~ (e^x - 1) / x on x in [-0.5, 0.5] (Chebyshev nodes).

The zero-order-hold write term of the kernels multiplies Delta*B*u by
(e^x - 1) / x with x = Delta * A. For |x| < 0.5 the kernels evaluate this
polynomial (no cancellation in e^x - 1); outside they use (e^x - 1) / x with the
exponential they already have. Q(0) is constrained to 1 so that x -> 0 gives
exactly the Delta*B*u limit. Run to regenerate the coefficients in
vscan_common.cuh and to print the relative error (float64 and float32 Horner).
"""
import numpy as np


def target(x):
    return np.where(x == 0, 1.0, np.expm1(x) / np.where(x == 0, 1.0, x))


def fit(degree, nodes=4000):
    k = np.arange(nodes)
    x = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)
    f = target(x)
    V = np.vander(x, degree + 1, increasing=True)[:, 1:]
    c, *_ = np.linalg.lstsq(V / f[:, None], (f - 1.0) / f, rcond=None)
    return np.concatenate([[1.0], c])


def rel_err(c, fp32=False):
    x = np.linspace(-0.5, 0.5, 400001)
    if fp32:
        x32 = x.astype(np.float32)
        acc = np.float32(c[-1])
        for ci in c[-2::-1]:
            acc = (acc * x32 + np.float32(ci)).astype(np.float32)
        p, x = acc.astype(np.float64), x32.astype(np.float64)
    else:
        p = np.polyval(c[::-1], x)
    return float(np.max(np.abs(p - target(x)) / target(x)))


if __name__ == "__main__":
    for d in range(4, 8):
        c = fit(d)
        print(f"degree {d}: rel err {rel_err(c):.2e} (fp64)  {rel_err(c, True):.2e} (fp32 Horner)")
    c = fit(6)
    print("coefficients, degree 6, c0..c6:")
    for ci in c:
        print(f"    {float(np.float32(ci)):.9e}f,")
