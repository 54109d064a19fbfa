"""Pins that tie the fp64 oracle to the pages and to mathematics, not to itself.

Each test checks the oracle against something fixed outside it: a value the
pages print (golden fixtures, with citations), a closed form, a textbook or
library routine (cumulative sums, means), or a structural invariant the pages
state (gather/merge round trips, visit counts, locality). The set is chosen so
that a dropped term, a wrong sign, a wrong index or a transposed operand in the
oracle fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest

from conftest import read_golden, read_route_fixture

import oracle as O


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- scalar recurrence
def test_worked_scalar_update_from_the_vim_page():
    """Vim review, "A state retains, writes, and reads": 0.5 * 2 + 0.2 * 3 = 1.6."""
    prev, keep, inp, write, new = map(float, read_golden("worked_scalar_update.txt")[0].split())
    # step 0 builds the previous state from zero: dt * B * u = 1 * prev * 1
    # step 1: retention e^{dt A} = keep with dt = 1, A = ln(keep); write dt * B = write
    y = O.scan_sequence(u=[1.0, inp], dt=[1.0, 1.0], A=[math.log(keep)],
                        B=[[prev], [write]], C=[[1.0], [1.0]], D=0.0)
    assert y[0] == pytest.approx(prev, abs=1e-15)
    assert y[1] == pytest.approx(new, abs=1e-14)


@pytest.mark.parametrize("L,N,seed", [(1, 1, 1), (3, 2, 2), (5, 3, 3), (8, 3, 4), (7, 1, 5)])
def test_recurrence_matches_unrolled_closed_form(L, N, seed):
    """h_t = sum_{s<=t} (prod_{r=s+1..t} e^{dt_r A}) dt_s B_s u_s, written as explicit products."""
    r = _rng(seed)
    u = r.standard_normal(L)
    dt = r.uniform(0.05, 1.5, L)
    A = -r.uniform(0.1, 3.0, N)
    B = r.standard_normal((L, N))
    C = r.standard_normal((L, N))
    D = r.standard_normal()
    y = O.scan_sequence(u, dt, A, B, C, D)
    for t in range(L):
        total = D * u[t]
        for n in range(N):
            h = 0.0
            for s in range(t + 1):
                prod = 1.0
                for q in range(s + 1, t + 1):
                    prod *= math.exp(dt[q] * A[n])
                h += prod * dt[s] * B[s, n] * u[s]
            total += C[t, n] * h
        assert y[t] == pytest.approx(total, rel=1e-12, abs=1e-14)


def test_impulse_response_is_analytic_decay():
    """u = delta_0: y_t = sum_n C_tn exp(A_n sum_{r=1..t} dt_r) dt_0 B_0n for t >= 1."""
    r = _rng(7)
    L, N = 12, 4
    u = np.zeros(L)
    u[0] = 1.0
    dt = r.uniform(0.01, 0.8, L)
    A = -np.arange(1, N + 1, dtype=float)
    B = r.standard_normal((L, N))
    C = r.standard_normal((L, N))
    y = O.scan_sequence(u, dt, A, B, C, D=0.7)
    assert y[0] == pytest.approx(np.dot(C[0], dt[0] * B[0]) + 0.7, rel=1e-13)
    for t in range(1, L):
        decay = np.exp(A * dt[1:t + 1].sum())
        assert y[t] == pytest.approx(np.dot(C[t], decay * dt[0] * B[0]), rel=1e-12)


def test_zero_decay_limit_is_a_cumulative_sum():
    """A = 0: retention 1, so h_t = sum_s dt_s B_s u_s (numpy cumsum)."""
    r = _rng(8)
    L = 20
    u = r.standard_normal(L)
    y = O.scan_sequence(u, np.ones(L), [0.0], np.ones((L, 1)), np.ones((L, 1)), D=0.0)
    np.testing.assert_allclose(y, np.cumsum(u), rtol=1e-13, atol=1e-13)


def test_full_forgetting_limit_keeps_only_the_current_write():
    """e^{dt A} = 0: y_t = C_t . (dt_t B_t u_t) + D u_t."""
    r = _rng(9)
    L, N = 10, 3
    u, dt = r.standard_normal(L), r.uniform(0.5, 1.0, L)
    B, C = r.standard_normal((L, N)), r.standard_normal((L, N))
    y = O.scan_sequence(u, dt, [-1e6] * N, B, C, D=-0.3)
    expect = np.einsum("tn,tn->t", C, dt[:, None] * B * u[:, None]) - 0.3 * u
    np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- routes
def test_atrous_routes_match_the_hand_derived_fixture():
    for (h, w), groups in read_route_fixture("atrous_routes.txt").items():
        got = O.route("atrous2", h, w)
        for k, idx in groups.items():
            assert got[k].tolist() == idx, (h, w, k)


def test_cross_scan_routes_match_the_hand_derived_fixture():
    for (h, w), groups in read_route_fixture("cross_scan_routes.txt").items():
        got = O.route("cross4", h, w)
        for k, idx in groups.items():
            assert got[k].tolist() == idx, (h, w, k)


def test_visit_counts_from_the_efficientvmamba_page():
    for ln in read_golden("visit_counts.txt"):
        h, w, dense, sparse, pad = map(int, ln.split())
        K, L, T = O.geometry("atrous2", h, w)
        K4, L4, _ = O.geometry("cross4", h, w)
        assert K4 * L4 == dense
        assert K * L == sparse
        assert int((O.route("atrous2", h, w) < 0).sum()) == pad


def test_vim_sequence_lengths_and_middle_cls():
    for ln in read_golden("vim_sequence_lengths.txt"):
        h, w, cls, tokens = map(int, ln.split())
        K, L, T = O.geometry("bidir", h, w, cls)
        assert (K, L, T) == (2, tokens, tokens)
        with pytest.raises(ValueError):
            O.geometry("bidir", h, w, cls + 1)


@pytest.mark.parametrize("h,w", [(1, 1), (1, 7), (7, 1), (2, 2), (3, 5), (5, 3), (4, 6),
                                 (6, 4), (9, 8), (8, 9), (11, 13)])
def test_routes_are_permutations_of_the_grid(h, w):
    """Atrous streams partition the real pixels (one owner each); every SS2D and bidirectional
    direction visits every token exactly once."""
    a = O.route("atrous2", h, w)
    real = a[a >= 0]
    assert sorted(real.tolist()) == list(range(h * w))
    assert a.shape == (4, ((h + 1) // 2) * ((w + 1) // 2))
    c = O.route("cross4", h, w)
    for k in range(4):
        assert sorted(c[k].tolist()) == list(range(h * w))
    b = O.route("bidir", h, w)
    assert b[1].tolist() == b[0][::-1].tolist()


# ---------------------------------------------------------------- routed forward
def _inputs(b, T, D, N, seed, K=None):
    r = _rng(seed)
    lead = () if K is None else (K,)
    return dict(u=r.standard_normal(lead + (b, T, D)), delta=0.5 * r.standard_normal(lead + (b, T, D)),
                B=r.standard_normal(lead + (b, T, N)), C=r.standard_normal(lead + (b, T, N)),
                z=r.standard_normal((b, T, D)))


@pytest.mark.parametrize("h,w", [(1, 1), (3, 5), (5, 3), (4, 6), (2, 7), (7, 2)])
def test_identity_operator_round_trips(h, w):
    """With B = C = 0 and D = 1 the scan returns u. Atrous gather+merge then gives X (not 4X);
    SS2D sums four aligned copies (4X); the bidirectional route two (2X)."""
    b, D, N = 2, 3, 4
    x = _inputs(b, h * w, D, N, 11)
    zeros = np.zeros((b, h * w, N))
    common = dict(A=-np.ones((D, N)), B=zeros, C=zeros, Dskip=np.ones(D), bias=np.zeros(D))
    ya = O.forward("atrous2", h, w, x["u"], x["delta"], **common)
    np.testing.assert_array_equal(ya, x["u"])
    yc = O.forward("cross4", h, w, x["u"], x["delta"], **common)
    np.testing.assert_allclose(yc, 4 * x["u"], rtol=0, atol=1e-15)
    yb = O.forward("bidir", h, w, x["u"], x["delta"], **common)
    np.testing.assert_allclose(yb, 2 * x["u"], rtol=0, atol=1e-15)


def _cumsum_operator(kind, h, w, u, cls=-1):
    """Run the oracle as a running-sum operator: A = 0, B = C = 1, dt = 1, D = 0."""
    b, T, D = u.shape
    ones = np.ones((b, T, 1))
    return O.forward(kind, h, w, u, np.ones_like(u), A=np.zeros((D, 1)), B=ones, C=ones,
                     Dskip=np.zeros(D), bias=None, cls_pos=cls, delta_softplus=False)


def test_bidirectional_running_sum_is_prefix_plus_suffix():
    h, w, cls = 3, 5, 7
    u = _rng(12).standard_normal((2, h * w + 1, 3))
    y = _cumsum_operator("bidir", h, w, u, cls)
    expect = np.cumsum(u, axis=1) + np.cumsum(u[:, ::-1], axis=1)[:, ::-1]
    np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("h,w", [(3, 5), (5, 3), (4, 4)])
def test_cross_scan_running_sum_uses_row_and_column_orders(h, w):
    u = _rng(13).standard_normal((1, h * w, 2))
    y = _cumsum_operator("cross4", h, w, u)
    g = u.reshape(1, h, w, 2)
    row = g.reshape(1, h * w, 2)
    col = g.transpose(0, 2, 1, 3).reshape(1, h * w, 2)  # column-major sequence
    pr = np.cumsum(row, 1) + np.cumsum(row[:, ::-1], 1)[:, ::-1]
    pc = np.cumsum(col, 1) + np.cumsum(col[:, ::-1], 1)[:, ::-1]
    pc_grid = pc.reshape(1, w, h, 2).transpose(0, 2, 1, 3).reshape(1, h * w, 2)
    np.testing.assert_allclose(y, pr + pc_grid, rtol=1e-13, atol=1e-12)


def test_atrous_running_sum_follows_the_fixture_order_through_padding():
    """Running sums along each hand-derived stream (padding contributes 0)."""
    for (h, w), groups in read_route_fixture("atrous_routes.txt").items():
        u = _rng(14).standard_normal((1, h * w, 1))
        y = _cumsum_operator("atrous2", h, w, u)
        expect = np.zeros(h * w)
        for k, idx in groups.items():
            vals = [u[0, i, 0] if i >= 0 else 0.0 for i in idx]
            run = np.cumsum(vals)
            for i, v in zip(idx, run):
                if i >= 0:
                    expect[i] = v
        np.testing.assert_allclose(y[0, :, 0], expect, rtol=1e-13, atol=1e-13)


def test_softplus_of_the_bias_recovers_dt0():
    """bias = log(expm1(dt0)) and raw delta = 0 give delta = softplus(bias) = dt0; softplus(0) = ln 2."""
    dt0 = np.array([1e-3, 0.05, 0.1, 2.0])
    D = dt0.size
    u = np.zeros((1, 1, D))
    u[0, 0] = 1.0
    one = np.ones((1, 1, 1))
    for bias, expect in ((np.log(np.expm1(dt0)), dt0), (np.zeros(D), np.full(D, math.log(2.0)))):
        # 1x1 grid, bidirectional: both directions see the single token, so y = 2 * delta
        y = O.forward("bidir", 1, 1, u, np.zeros_like(u), A=np.zeros((D, 1)), B=one, C=one,
                      Dskip=np.zeros(D), bias=bias)
        np.testing.assert_allclose(y[0, 0], 2 * expect, rtol=1e-13)


def test_backward_direction_is_forward_scan_of_the_reversed_sequence():
    """Vim: bwd(x) = flip(fwd(flip(x))), isolated by giving direction 0 zero input and no skip."""
    h, w, D, N = 3, 4, 2, 3
    x = _inputs(1, h * w, D, N, 15, K=2)
    x["u"][0] = 0.0
    r = _rng(16)
    A = -r.uniform(0.2, 2.0, (2, D, N))
    Dsk = np.stack([np.zeros(D), r.standard_normal(D)])
    bias = r.standard_normal((2, D)) * 0.1
    y = O.forward("bidir", h, w, x["u"], x["delta"], A, x["B"], x["C"], Dsk, bias,
                  per_dir_inputs=True, per_dir_params=True)
    for d in range(D):
        sp = np.logaddexp(0.0, x["delta"][1, 0, :, d] + bias[1, d])  # numpy softplus
        rev = O.scan_sequence(x["u"][1, 0, ::-1, d], sp[::-1], A[1, d], x["B"][1, 0, ::-1],
                              x["C"][1, 0, ::-1], Dsk[1, d])
        np.testing.assert_allclose(y[0, :, d], rev[::-1], rtol=1e-12, atol=1e-14)


def test_atrous_groups_do_not_read_each_other():
    """EfficientVMamba: an even/even state never reads an odd/odd feature. Perturbing one pixel
    changes outputs only inside that pixel's stream, at or after it."""
    h, w, D, N = 5, 6, 2, 4
    x = _inputs(1, h * w, D, N, 17)
    A = -np.arange(1, N + 1, dtype=float)[None].repeat(D, 0)
    base = O.forward("atrous2", h, w, x["u"], x["delta"], A, x["B"], x["C"], np.ones(D), np.zeros(D))
    routes = O.route("atrous2", h, w)
    for k in range(4):
        stream = [i for i in routes[k] if i >= 0]
        p = stream[1]
        x2 = {kk: v.copy() for kk, v in x.items()}
        x2["u"][0, p] += 1.0
        y2 = O.forward("atrous2", h, w, x2["u"], x2["delta"], A, x2["B"], x2["C"], np.ones(D), np.zeros(D))
        changed = set(np.nonzero(np.any(y2[0] != base[0], axis=1))[0].tolist())
        assert changed and changed <= set(stream[1:]), (k, changed)


def test_pooled_route_is_the_bidirectional_scan_of_axis_means():
    """FastVim: mean-pool (numpy mean) then scan both ways, then repeat over the pooled axis."""
    h, w, D, N = 4, 5, 3, 2
    x = _inputs(2, h * w, D, N, 18)
    A = -_rng(19).uniform(0.5, 2.0, (D, N))
    bias = _rng(20).standard_normal(D) * 0.3
    y = O.forward("pool_w", h, w, x["u"], x["delta"], A, x["B"], x["C"], np.ones(D), bias)
    for kind, axis, L in (("pool_w", 2, h), ("pool_h", 1, w)):
        y = O.forward(kind, h, w, x["u"], x["delta"], A, x["B"], x["C"], np.ones(D), bias)
        pool = {k: x[k].reshape(2, h, w, -1).mean(axis=axis) for k in ("u", "delta", "B", "C")}
        ref = O.forward("bidir", L, 1, pool["u"], pool["delta"], A, pool["B"], pool["C"], np.ones(D), bias)
        grid = y.reshape(2, h, w, D)
        if kind == "pool_w":
            np.testing.assert_allclose(grid, np.repeat(ref[:, :, None], w, axis=2), rtol=1e-12, atol=1e-13)
        else:
            np.testing.assert_allclose(grid, np.repeat(ref[:, None], h, axis=1), rtol=1e-12, atol=1e-13)


def test_pool_h_is_pool_w_on_the_transposed_grid():
    h, w, D, N = 3, 6, 2, 3
    x = _inputs(1, h * w, D, N, 21)
    A = -np.ones((D, N)) * np.arange(1, N + 1)
    yh = O.forward("pool_h", h, w, x["u"], x["delta"], A, x["B"], x["C"], np.ones(D), np.zeros(D), z=x["z"])
    t = {k: x[k].reshape(1, h, w, -1).transpose(0, 2, 1, 3).reshape(1, h * w, -1)
         for k in ("u", "delta", "B", "C", "z")}
    yw = O.forward("pool_w", w, h, t["u"], t["delta"], A, t["B"], t["C"], np.ones(D), np.zeros(D), z=t["z"])
    back = yw.reshape(1, w, h, D).transpose(0, 2, 1, 3).reshape(1, h * w, D)
    np.testing.assert_allclose(yh, back, rtol=1e-13, atol=1e-14)


def test_gate_merge_scale_and_shared_parameters():
    h, w, D, N = 3, 3, 4, 2
    x = _inputs(1, h * w, D, N, 22)
    A = -_rng(23).uniform(0.5, 2.0, (D, N))
    Dsk, bias = np.ones(D), np.zeros(D)
    for kind in ("bidir", "cross4", "atrous2", "pool_w"):
        y1 = O.forward(kind, h, w, x["u"], x["delta"], A, x["B"], x["C"], Dsk, bias)
        yh = O.forward(kind, h, w, x["u"], x["delta"], A, x["B"], x["C"], Dsk, bias, merge_scale=0.5)
        np.testing.assert_allclose(yh, 0.5 * y1, rtol=1e-15)
        yz0 = O.forward(kind, h, w, x["u"], x["delta"], A, x["B"], x["C"], Dsk, bias, z=np.zeros_like(x["z"]))
        assert np.all(yz0 == 0.0)
        yzb = O.forward(kind, h, w, x["u"], x["delta"], A, x["B"], x["C"], Dsk, bias, z=np.full_like(x["z"], 60.0))
        np.testing.assert_allclose(yzb, 60.0 * y1, rtol=1e-13)
        yg = O.forward(kind, h, w, x["u"], x["delta"], A, x["B"], x["C"], Dsk, bias, z=x["z"])
        np.testing.assert_allclose(yg, y1 * x["z"] / (1 + np.exp(-x["z"])), rtol=1e-13, atol=1e-15)
        K = 4 if kind in ("cross4", "atrous2") else 2
        rep = lambda a: np.broadcast_to(a, (K,) + a.shape).copy()
        yp = O.forward(kind, h, w, rep(x["u"]), rep(x["delta"]), rep(A), rep(x["B"]), rep(x["C"]),
                       rep(Dsk), rep(bias), per_dir_inputs=True, per_dir_params=True)
        np.testing.assert_array_equal(yp, y1)


def test_channels_and_images_are_independent():
    """Slicing channels or images before the oracle equals slicing its output."""
    import workloads
    wl = workloads.WORKLOADS["evmamba_atrous_55x57"].with_(batch=2, D=8)
    x = workloads.draw(wl)
    full = O.forward(wl.route, wl.h, wl.w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"], x["z"])
    xs = workloads.batch_slice(workloads.channel_slice(x, [1, 6]), [1])
    part = O.forward(wl.route, wl.h, wl.w, xs["u"], xs["delta"], xs["A"], xs["B"], xs["C"], xs["Dskip"], xs["bias"], xs["z"])
    np.testing.assert_array_equal(part, full[1:2][..., [1, 6]])


# ---------------------------------------------------------------- padding is a real step
def _atrous_stream(h, w, k):
    """Grid coordinates of atrous group k in visiting order, written out from the EfficientVMamba
    review, sec. 1: offsets (m, n) = (0,0), (1,0), (0,1), (1,1) in (row, column); groups 0 and 2
    row-major, 1 and 3 column-major, on the grid padded right/bottom to even size. A coordinate
    outside h x w is a padding slot (None)."""
    m, n = k & 1, k >> 1
    rows, cols = (h + 1) // 2, (w + 1) // 2
    order = [(r, c) for c in range(cols) for r in range(rows)] if k & 1 else \
            [(r, c) for r in range(rows) for c in range(cols)]
    out = []
    for r, c in order:
        y, x = 2 * r + m, 2 * c + n
        out.append(y * w + x if (y < h and x < w) else None)
    return out


def _pad_runs(stream):
    """(source token, pads skipped, next token) for every real token followed by padding and then
    by another real token of the same stream."""
    runs = []
    for i, p in enumerate(stream):
        if p is None or i + 1 >= len(stream) or stream[i + 1] is not None:
            continue
        j = i + 1
        while j < len(stream) and stream[j] is None:
            j += 1
        if j < len(stream):
            runs.append((p, j - i - 1, stream[j]))
    return runs


@pytest.mark.parametrize("h,w,samples", [(3, 5, None), (5, 3, None), (55, 57, 6)])
def test_padding_slots_decay_the_state(h, w, samples):
    """EfficientVMamba review, sec. 1-2: padding positions are zero-valued inputs to the scan, not
    absent steps, so the state keeps decaying across them. With u an impulse at the last real token
    before a run of k pads, the next real token of that stream reads
        y = sum_n C_n exp(A_n (k softplus(bias) + softplus(raw_next + bias))) softplus(raw_src + bias) B_src,n.
    Skipping the pads, or giving them Delta = 0, drops the k softplus(bias) term."""
    r = _rng(31)
    N = 3
    A = -np.array([[0.7, 1.9, 3.1]])
    bias = np.array([0.4])  # softplus(0.4) = 0.913: a pad decays exp(-0.64 .. -2.8) per step
    sp = lambda v: np.logaddexp(0.0, v)  # noqa: E731  (numpy softplus)
    checked = 0
    for k in range(4):
        runs = _pad_runs(_atrous_stream(h, w, k))
        if samples is not None:
            runs = runs[:: max(1, len(runs) // samples)][:samples]
        for src, npad, nxt in runs:
            raw = 0.5 * r.standard_normal((1, h * w, 1))
            B = r.standard_normal((1, h * w, N))
            C = r.standard_normal((1, h * w, N))
            u = np.zeros((1, h * w, 1))
            u[0, src, 0] = 1.0
            y = O.forward("atrous2", h, w, u, raw, A, B, C, Dskip=np.zeros(1), bias=bias)
            decay = np.exp(A[0] * (npad * sp(bias[0]) + sp(raw[0, nxt, 0] + bias[0])))
            expect = np.dot(C[0, nxt], decay * sp(raw[0, src, 0] + bias[0]) * B[0, src])
            assert y[0, nxt, 0] == pytest.approx(expect, rel=1e-12, abs=1e-15), (k, src, npad, nxt)
            # the same impulse with the pads removed would read a visibly different value
            no_pad = np.dot(C[0, nxt], np.exp(A[0] * sp(raw[0, nxt, 0] + bias[0]))
                            * sp(raw[0, src, 0] + bias[0]) * B[0, src])
            assert abs(no_pad - expect) > 1e-3 * max(abs(expect), 1e-3)
            checked += 1
    assert checked >= 3
