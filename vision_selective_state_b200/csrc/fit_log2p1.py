"""Least-squares fit of P(t) ~ log2(1 + t) / t on t in [0, 1] (Chebyshev nodes).

The kernels evaluate softplus(x) = max(x, 0) + ln2 * t * P(t), t = 2^(-|x| log2 e),
which is the identity softplus(x) = max(x, 0) + log(1 + e^-|x|) with the log
replaced by this polynomial. Run to regenerate the coefficients in
vscan_common.cuh and to print the fit's relative error (float64 and float32
Horner evaluation).
"""
import numpy as np


def fit(degree, nodes=4000):
    k = np.arange(nodes)
    t = 0.5 - 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [0, 1]
    f = np.log2(1 + t) / t
    # weight by 1/f so the residual is a relative error of log2(1 + t)
    V = np.vander(t, degree + 1, increasing=True)
    c, *_ = np.linalg.lstsq(V / f[:, None], np.ones_like(f), rcond=None)
    return c


def rel_err(c, fp32=False):
    t = np.linspace(1e-9, 1.0, 200001)
    if fp32:
        t32 = t.astype(np.float32)
        acc = np.float32(c[-1])
        for ci in c[-2::-1]:
            acc = (acc * t32 + np.float32(ci)).astype(np.float32)
        p = acc.astype(np.float64)
        t = t32.astype(np.float64)
    else:
        p = np.polyval(c[::-1], t)
    exact = np.log2(1 + t) / t
    return float(np.max(np.abs(p - exact) / exact))


if __name__ == "__main__":
    for d in range(5, 11):
        c = fit(d)
        print(f"degree {d}: rel err {rel_err(c):.2e} (fp64)  {rel_err(c, True):.2e} (fp32 Horner)")
    c = fit(8)
    print("coefficients, degree 8, c0..c8:")
    for ci in c:
        print(f"    {float(np.float32(ci)):.9e}f,")
