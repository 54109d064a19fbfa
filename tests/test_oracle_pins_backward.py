"""Pins for the oracle's backward pass: every gradient equals the central finite
difference of the (separately pinned) forward oracle, entry by entry, on tiny
inputs of every route, with shared and per-direction inputs and parameters,
with and without the gate, skip term, bias and softplus. Finite differences
are the definition of the derivative, independent of the reverse-mode code.
"""
import numpy as np
import pytest

import oracle as O

EPS = 1e-6


def _inputs(kind, h, w, cls, pdi, pdp, seed, D=2, N=3, b=2):
    K, L, T = O.geometry(kind, h, w, cls)
    r = np.random.default_rng(seed)
    li = (K,) if pdi else ()
    lp = (K,) if pdp else ()
    return dict(u=r.standard_normal(li + (b, T, D)), delta=0.5 * r.standard_normal(li + (b, T, D)),
                B=r.standard_normal(li + (b, T, N)), C=r.standard_normal(li + (b, T, N)),
                A=-np.exp(0.3 * r.standard_normal(lp + (D, N))) * np.arange(1, N + 1),
                Dskip=r.standard_normal(lp + (D,)), bias=0.3 * r.standard_normal(lp + (D,)),
                z=r.standard_normal((b, T, D))), r.standard_normal((b, T, D))


def _loss(kind, h, w, cls, x, dy, **kw):
    y = O.forward(kind, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"], x["z"],
                  cls_pos=cls, **kw)
    return float(np.sum(y * dy))


@pytest.mark.parametrize("kind,h,w,cls", [("bidir", 2, 3, 3), ("bidir", 1, 4, -1), ("cross4", 2, 3, -1),
                                          ("atrous2", 3, 3, -1), ("atrous2", 2, 4, -1), ("pool_w", 3, 4, -1),
                                          ("pool_h", 3, 2, -1)])
@pytest.mark.parametrize("pdi,pdp", [(False, False), (True, True)])
def test_gradients_equal_finite_differences(kind, h, w, cls, pdi, pdp):
    x, dy = _inputs(kind, h, w, cls, pdi, pdp, seed=hash((kind, h, w)) % 1000)
    kw = dict(per_dir_inputs=pdi, per_dir_params=pdp, merge_scale=0.7)
    g = O.backward(kind, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"], x["z"],
                   dy=dy, cls_pos=cls, **kw)
    names = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "Dskip": "dDskip",
             "bias": "dbias", "z": "dz"}
    for key, gk in names.items():
        fd = np.empty_like(x[key])
        for idx in np.ndindex(x[key].shape):
            xp = {k: v.copy() for k, v in x.items()}
            xm = {k: v.copy() for k, v in x.items()}
            xp[key][idx] += EPS
            xm[key][idx] -= EPS
            fd[idx] = (_loss(kind, h, w, cls, xp, dy, **kw) - _loss(kind, h, w, cls, xm, dy, **kw)) / (2 * EPS)
        np.testing.assert_allclose(g[gk], fd, rtol=1e-5, atol=1e-7, err_msg=f"{kind} {key}")


@pytest.mark.parametrize("kind,h,w,cls", [("bidir", 2, 3, -1), ("atrous2", 3, 3, -1), ("pool_w", 2, 3, -1)])
def test_gradients_without_optional_terms(kind, h, w, cls):
    """No gate, no skip, no bias, no softplus: the same finite-difference check."""
    x, dy = _inputs(kind, h, w, cls, False, False, seed=7)
    x["delta"] = np.abs(x["delta"]) + 0.05
    def loss(xx):
        y = O.forward(kind, h, w, xx["u"], xx["delta"], xx["A"], xx["B"], xx["C"], cls_pos=cls,
                      delta_softplus=False)
        return float(np.sum(y * dy))
    g = O.backward(kind, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"], dy=dy, cls_pos=cls,
                   delta_softplus=False)
    for key, gk in (("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC")):
        fd = np.empty_like(x[key])
        for idx in np.ndindex(x[key].shape):
            xp = {k: v.copy() for k, v in x.items()}
            xm = {k: v.copy() for k, v in x.items()}
            xp[key][idx] += EPS
            xm[key][idx] -= EPS
            fd[idx] = (loss(xp) - loss(xm)) / (2 * EPS)
        np.testing.assert_allclose(g[gk], fd, rtol=1e-5, atol=1e-7, err_msg=f"{kind} {key}")
    # without a skip term or bias the corresponding gradients are still defined (w.r.t. zero)
    assert np.all(np.isfinite(g["dDskip"])) and np.all(np.isfinite(g["dbias"]))
