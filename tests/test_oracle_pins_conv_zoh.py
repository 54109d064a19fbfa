"""Pins for the two optional steps of the oracle: the fused causal convolution
and the zero-order-hold write term.

Convolution: [Vim] "Inside the released Vim block" (each direction runs its own
kernel-four causal Conv1d, then SiLU, the backward one on the reversed
sequence) and "CPU backend substitutions" (a grouped conv1d with left padding);
[FVim] Methodology (Conv1D, then mean-pool one axis). Pinned against
numpy.convolve along each direction's order, fed to the un-convolved oracle.

Zero-order hold: [NoD] Eq. 2, Bbar = (dt A)^-1 (exp(dt A) - I) dt B, i.e. the
exact solution of h' = A h + B u over an interval of length dt with u and B
held constant. Pinned against a Runge-Kutta integration of that ODE.
"""
import numpy as np
import pytest

import oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


def _silu(x):
    return x / (1.0 + np.exp(-x))


def _causal(x, w, b):
    """SiLU(b + sum_i w[i] x[t - 3 + i]) along axis 0 by numpy.convolve (x[<0] = 0)."""
    out = np.empty_like(x)
    for d in range(x.shape[1]):
        out[:, d] = np.convolve(x[:, d], w[d][::-1])[: x.shape[0]] + b[d]
    return _silu(out)


def _inputs(b, T, D, N, seed):
    r = _rng(seed)
    return dict(x=r.standard_normal((b, T, D)), delta=0.5 * r.standard_normal((b, T, D)),
                B=r.standard_normal((b, T, N)), C=r.standard_normal((b, T, N)),
                A=-np.exp(0.3 * r.standard_normal((D, N))) * np.arange(1, N + 1),
                Dskip=r.standard_normal(D), bias=np.log(np.expm1(r.uniform(1e-3, 0.1, D))),
                z=r.standard_normal((b, T, D)))


def _order(kind, h, w, k, T):
    """Token visited at each step of direction k's convolution order."""
    if kind == "bidir":
        base = np.arange(T)
    elif kind == "pool_w":
        base = np.arange(h * w)                      # row-major
    else:
        s = np.arange(h * w)
        base = (s % h) * w + s // h                  # column-major
    return base if k == 0 else base[::-1]


@pytest.mark.parametrize("kind,h,w,cls", [("bidir", 3, 5, 7), ("bidir", 4, 4, -1),
                                          ("pool_w", 5, 7, -1), ("pool_h", 5, 7, -1),
                                          ("pool_w", 1, 1, -1), ("bidir", 1, 1, -1)])
@pytest.mark.parametrize("per_dir_params", [False, True])
def test_conv_equals_numpy_convolution_along_each_direction(kind, h, w, cls, per_dir_params):
    K, L, T = O.geometry(kind, h, w, cls)
    D, N, b = 3, 4, 2
    x = _inputs(b, T, D, N, seed=11)
    r = _rng(12)
    shape_w, shape_b = ((K, D, 4), (K, D)) if per_dir_params else ((D, 4), (D,))
    cw, cb = r.standard_normal(shape_w), r.standard_normal(shape_b)
    A = np.stack([x["A"], 0.7 * x["A"]]) if per_dir_params else x["A"]
    Dk = np.stack([x["Dskip"], -x["Dskip"]]) if per_dir_params else x["Dskip"]
    bias = np.stack([x["bias"], x["bias"] + 0.1]) if per_dir_params else x["bias"]
    got = O.forward(kind, h, w, x["x"], x["delta"], A, x["B"], x["C"], Dk, bias, x["z"],
                    cls_pos=cls, per_dir_params=per_dir_params, conv_w=cw, conv_b=cb)
    # reference: convolve with numpy along each direction's order, then run the
    # oracle without convolution on per-direction inputs
    u = np.empty((K, b, T, D))
    for k in range(K):
        wk = cw[k] if per_dir_params else cw
        bk = cb[k] if per_dir_params else cb
        order = _order(kind, h, w, k, T)
        for i in range(b):
            u[k, i, order] = _causal(x["x"][i, order], wk, bk)
    rep = lambda a: np.stack([a] * K)
    ref = O.forward(kind, h, w, u, rep(x["delta"]), A, rep(x["B"]), rep(x["C"]), Dk, bias,
                    x["z"], cls_pos=cls, per_dir_inputs=True, per_dir_params=per_dir_params)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind,h,w,cls", [("bidir", 3, 5, 7), ("pool_w", 4, 6, -1), ("pool_h", 4, 6, -1)])
def test_identity_kernel_is_an_elementwise_silu(kind, h, w, cls):
    K, L, T = O.geometry(kind, h, w, cls)
    D, N, b = 2, 3, 1
    x = _inputs(b, T, D, N, seed=21)
    cw = np.zeros((D, 4)); cw[:, 3] = 1.0
    got = O.forward(kind, h, w, x["x"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"],
                    x["z"], cls_pos=cls, conv_w=cw, conv_b=np.zeros(D))
    ref = O.forward(kind, h, w, _silu(x["x"]), x["delta"], x["A"], x["B"], x["C"], x["Dskip"],
                    x["bias"], x["z"], cls_pos=cls)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


def test_shift_kernel_delays_the_forward_branch_and_advances_the_backward_one():
    """w = [0, 0, 1, 0]: the forward branch sees the previous token, the backward
    branch (reversed order) the next one; the first step of each sees zero."""
    h, w = 1, 6
    T = 6
    D, N = 1, 1
    x = np.arange(1.0, T + 1).reshape(1, T, 1)
    cw = np.array([[0.0, 0.0, 1.0, 0.0]])
    # scan that passes u straight through: A -> -inf kills the state, C = 0, D = 1
    ones = np.ones((1, T, N))
    got = O.forward("bidir", h, w, x, np.zeros((1, T, 1)), [[-1e9]], ones, 0 * ones, [1.0],
                    conv_w=cw, conv_b=[0.0], delta_softplus=False)
    fwd = _silu(np.array([0.0, 1, 2, 3, 4, 5]))
    bwd = _silu(np.array([2.0, 3, 4, 5, 6, 0]))
    np.testing.assert_allclose(got[0, :, 0], fwd + bwd, rtol=1e-14)


@pytest.mark.parametrize("kind", ["atrous2", "cross4"])
def test_conv_is_refused_on_grid_routes(kind):
    x = _inputs(1, 16, 2, 2, seed=3)
    with pytest.raises(RuntimeError):
        O.forward(kind, 4, 4, x["x"], x["delta"], x["A"], x["B"], x["C"], conv_w=np.zeros((2, 4)))


# ------------------------------------------------------------------ zero-order hold
def _rk4_scan(u, dt, A, B, C, D, substeps=400):
    """Integrate h' = A h + B_t u_t over each interval t of length dt_t (u, B held),
    then read y_t = C_t . h + D u_t at the end of the interval."""
    N = A.shape[0]
    h = np.zeros(N)
    y = np.empty(len(u))
    for t in range(len(u)):
        f = lambda hh: A * hh + B[t] * u[t]
        s = dt[t] / substeps
        for _ in range(substeps):
            k1 = f(h); k2 = f(h + 0.5 * s * k1); k3 = f(h + 0.5 * s * k2); k4 = f(h + s * k3)
            h = h + s / 6.0 * (k1 + 2 * k2 + 2 * k3 + k4)
        y[t] = C[t] @ h + D * u[t]
    return y


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_zero_order_hold_is_the_exact_ode_solution(seed):
    r = _rng(100 + seed)
    L, N = 7, 3
    u, dt = r.standard_normal(L), r.uniform(0.05, 1.5, L)
    A = -r.uniform(0.2, 3.0, N)
    B, C = r.standard_normal((L, N)), r.standard_normal((L, N))
    ref = _rk4_scan(u, dt, A, B, C, 0.4)
    got = O.scan_sequence(u, dt, A, B, C, 0.4, zoh=True)
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-10)
    # the released dt*B*u write is a different (first-order) discretization
    assert np.max(np.abs(O.scan_sequence(u, dt, A, B, C, 0.4) - ref)) > 1e-3


def test_zero_order_hold_limit_at_a_zero_decay_rate():
    r = _rng(7)
    L, N = 5, 2
    u, dt = r.standard_normal(L), r.uniform(0.1, 1.0, L)
    B, C = r.standard_normal((L, N)), r.standard_normal((L, N))
    zero = O.scan_sequence(u, dt, [0.0, 0.0], B, C, zoh=True)
    np.testing.assert_array_equal(zero, O.scan_sequence(u, dt, [0.0, 0.0], B, C))
    tiny = O.scan_sequence(u, dt, [-1e-12, -1e-12], B, C, zoh=True)
    np.testing.assert_allclose(tiny, zero, rtol=1e-9, atol=1e-12)


def test_zero_order_hold_reaches_the_steady_state():
    """Constant input over a long interval: h -> -B u / A."""
    A, B, u = np.array([-2.0]), np.array([[3.0]]), np.array([0.5])
    y = O.scan_sequence(u, [60.0], A, B, np.array([[1.0]]), zoh=True)
    assert y[0] == pytest.approx(-3.0 * 0.5 / -2.0, rel=1e-14)


@pytest.mark.parametrize("kind,h,w,cls", [("bidir", 3, 4, 6), ("atrous2", 3, 5, -1),
                                          ("cross4", 2, 3, -1), ("pool_w", 3, 4, -1)])
def test_zero_order_hold_reaches_every_route(kind, h, w, cls):
    """forward(zoh) differs from forward() only through the write term: with
    A = 0 both are equal, with A != 0 they differ."""
    K, L, T = O.geometry(kind, h, w, cls)
    x = _inputs(1, T, 2, 3, seed=5)
    args = (kind, h, w, x["x"], x["delta"])
    rest = (x["B"], x["C"], x["Dskip"], x["bias"], x["z"])
    z0 = np.zeros_like(x["A"])
    np.testing.assert_array_equal(O.forward(*args, z0, *rest, cls_pos=cls, zoh=True),
                                  O.forward(*args, z0, *rest, cls_pos=cls))
    assert np.max(np.abs(O.forward(*args, x["A"], *rest, cls_pos=cls, zoh=True)
                         - O.forward(*args, x["A"], *rest, cls_pos=cls))) > 1e-6
