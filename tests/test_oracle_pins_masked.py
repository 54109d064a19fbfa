"""Pins for the masked pooled route (FastMaskVim: "Fast Vision Mamba ...",
"Innovation": sparse indexing for masked or irregular grids, row sums
normalized by the nominal width; "Methodology": mask-aware aggregation).

The masked oracle is pinned to the dense pooled oracle (itself pinned in
test_oracle_pins.py): with every token visible it is the dense route; the
order of the visible tokens does not matter; and a sparse set gives, at the
visible tokens, the dense result on the grid with the hidden tokens set to
zero (a zero token adds nothing to a row sum, and the divisor is the nominal
width either way).
"""
import numpy as np
import pytest

import oracle as O


def _dense(h, w, D, N, b, seed):
    r = np.random.default_rng(seed)
    T = h * w
    return dict(u=r.standard_normal((b, T, D)), delta=0.5 * r.standard_normal((b, T, D)),
                B=r.standard_normal((b, T, N)), C=r.standard_normal((b, T, N)),
                z=r.standard_normal((b, T, D)),
                A=-np.exp(0.3 * r.standard_normal((D, N))) * np.arange(1, N + 1),
                Dskip=r.standard_normal(D), bias=np.log(np.expm1(r.uniform(1e-3, 0.1, D))))


def _masked_call(kind, h, w, pos, x, sel, **kw):
    take = lambda a: np.stack([a[i, sel[i]] for i in range(a.shape[0])])
    return O.forward_masked(kind, h, w, pos, take(x["u"]), take(x["delta"]), x["A"], take(x["B"]),
                            take(x["C"]), x["Dskip"], x["bias"], take(x["z"]), **kw)


@pytest.mark.parametrize("kind", ["pool_w", "pool_h"])
@pytest.mark.parametrize("h,w", [(1, 1), (4, 6), (7, 3)])
def test_full_mask_is_the_dense_route(kind, h, w):
    x = _dense(h, w, 3, 4, 2, seed=1)
    T = h * w
    sel = [np.arange(T)] * 2
    pos = np.stack(sel)
    got = _masked_call(kind, h, w, pos, x, sel)
    ref = O.forward(kind, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"], x["z"])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["pool_w", "pool_h"])
def test_visible_token_order_does_not_matter(kind):
    h, w = 5, 6
    x = _dense(h, w, 2, 3, 1, seed=2)
    r = np.random.default_rng(3)
    sel = np.sort(r.choice(h * w, 11, replace=False))
    perm = r.permutation(11)
    a = _masked_call(kind, h, w, sel[None], x, [sel])
    b = _masked_call(kind, h, w, sel[perm][None], x, [sel[perm]])
    np.testing.assert_allclose(b[0], a[0][perm], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["pool_w", "pool_h"])
@pytest.mark.parametrize("h,w,keep", [(6, 8, 12), (9, 5, 1), (4, 4, 16), (8, 8, 16)])
@pytest.mark.parametrize("zoh", [False, True])
def test_sparse_set_equals_dense_grid_with_hidden_tokens_zeroed(kind, h, w, keep, zoh):
    b = 2
    x = _dense(h, w, 3, 5, b, seed=4)
    r = np.random.default_rng(5)
    sel = [np.sort(r.choice(h * w, keep, replace=False)) for _ in range(b)]
    pos = np.stack(sel)
    got = _masked_call(kind, h, w, pos, x, sel, zoh=zoh)
    xz = dict(x)
    for key in ("u", "delta", "B", "C"):
        dense = np.zeros_like(x[key])
        for i in range(b):
            dense[i, sel[i]] = x[key][i, sel[i]]
        xz[key] = dense
    ref = O.forward(kind, h, w, xz["u"], xz["delta"], x["A"], xz["B"], xz["C"], x["Dskip"], x["bias"],
                    x["z"], zoh=zoh)
    for i in range(b):
        np.testing.assert_allclose(got[i], ref[i, sel[i]], rtol=1e-12, atol=1e-12)


def test_row_sum_is_divided_by_the_nominal_width_not_the_count():
    """One visible token of value 1 in a row of width w pools to 1/w: with
    A -> -inf (no memory), C = B = 1, dt = 1 after softplus is off, the scan
    output of that row is C.B*dt*u/w... here isolated through the skip term
    D*u only (B = C = 0): y = 2 directions * D * u/w."""
    h, w = 3, 5
    pos = np.array([[7]])  # row 1, column 2
    u = np.ones((1, 1, 1))
    zero = np.zeros((1, 1, 2))
    y = O.forward_masked("pool_w", h, w, pos, u, np.zeros((1, 1, 1)), -np.ones((1, 2)), zero, zero,
                         Dskip=[1.0], delta_softplus=False)
    assert y[0, 0, 0] == pytest.approx(2.0 / w, rel=1e-15)
    y = O.forward_masked("pool_h", h, w, pos, u, np.zeros((1, 1, 1)), -np.ones((1, 2)), zero, zero,
                         Dskip=[1.0], delta_softplus=False)
    assert y[0, 0, 0] == pytest.approx(2.0 / h, rel=1e-15)


def test_positions_outside_the_grid_are_refused():
    with pytest.raises(RuntimeError):
        O.forward_masked("pool_w", 2, 2, [[4]], np.ones((1, 1, 1)), np.ones((1, 1, 1)), -np.ones((1, 1)),
                         np.ones((1, 1, 1)), np.ones((1, 1, 1)))
