"""fp64 CPU oracle for the routed visual selective scan.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py may import this package. It shares no
code with the CUDA library (vision_selective_state_b200) and never calls it.

The arithmetic lives in vscan_oracle.c (plain C, double precision); this module
only marshals numpy arrays into it. Each C function cites the page passage it
follows. Pins that tie the oracle to the pages are in tests/test_oracle_pins.py.
"""
import ctypes
import os

import numpy as np

from . import build as _build

BIDIR, CROSS4, ATROUS2, POOL_W, POOL_H = 0, 1, 2, 3, 4
ROUTE_NAMES = {"bidir": BIDIR, "cross4": CROSS4, "atrous2": ATROUS2,
               "pool_w": POOL_W, "pool_h": POOL_H}

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i = ctypes.c_int
        p = ctypes.c_void_p
        lib.oracle_geometry.argtypes = [i, i, i, i, p, p, p]
        lib.oracle_geometry.restype = i
        lib.oracle_route.argtypes = [i, i, i, i, p]
        lib.oracle_route.restype = i
        lib.oracle_scan_sequence.argtypes = [i, i, p, p, p, p, p, ctypes.c_double, i, p, p]
        lib.oracle_scan_sequence.restype = None
        lib.oracle_forward.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p, p, p, i,
                                       ctypes.c_double, i, i, p, p, i, p, i]
        lib.oracle_forward.restype = i
        lib.oracle_forward_masked.argtypes = [i, i, i, i, i, p, i, i, p, p, p, p, p, p, p, p, i,
                                              ctypes.c_double, i, i, i, p, i]
        lib.oracle_forward_masked.restype = i
        lib.oracle_backward.argtypes = [i, i, i, i, i, i, i, p, p, p, p, p, p, p, p, i, ctypes.c_double,
                                        i, i, p, p, p, p, p, p, p, p, p, i]
        lib.oracle_backward.restype = i
        lib.oracle_default_threads.argtypes = []
        lib.oracle_default_threads.restype = i
        _lib = lib
    return _lib


def _kind(kind):
    return ROUTE_NAMES[kind] if isinstance(kind, str) else int(kind)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return _load().oracle_default_threads()


def geometry(kind, h, w, cls_pos=-1):
    """(K, L, tokens) for a route, or raise ValueError."""
    K, L, T = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    rc = _load().oracle_geometry(_kind(kind), h, w, cls_pos, ctypes.byref(K),
                                 ctypes.byref(L), ctypes.byref(T))
    if rc != 0:
        raise ValueError(f"invalid route geometry (rc={rc})")
    return K.value, L.value, T.value


def route(kind, h, w, cls_pos=-1):
    """[K, L] int64 array: token (or pooled) index visited at each step, -1 = pad."""
    K, L, _ = geometry(kind, h, w, cls_pos)
    out = np.empty((K, L), dtype=np.int64)
    rc = _load().oracle_route(_kind(kind), h, w, cls_pos, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_route failed (rc={rc})")
    return out


def scan_sequence(u, dt, A, B, C, D=0.0, zoh=False):
    """One channel, one sequence: h_t = e^{dt_t A} h + dt_t B_t u_t, y_t = C_t.h_t + D u_t.

    u, dt: [L]; A: [N]; B, C: [L, N]. dt is already discretized. Returns y [L].
    zoh=True writes expm1(dt A) / A * B_t u_t (zero-order hold) instead of dt B_t u_t.
    """
    u, dt, A, B, C = map(_f64, (u, dt, A, B, C))
    L = u.shape[0]
    N = A.shape[0]
    assert dt.shape == (L,) and B.shape == (L, N) and C.shape == (L, N)
    y = np.empty(L, dtype=np.float64)
    h = np.empty(N, dtype=np.float64)
    _load().oracle_scan_sequence(L, N, _ptr(u), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                 float(D), int(bool(zoh)), _ptr(h), _ptr(y))
    return y


def forward(kind, h, w, u, delta, A, B, C, Dskip=None, bias=None, z=None, *,
            cls_pos=-1, delta_softplus=True, merge_scale=1.0,
            per_dir_inputs=False, per_dir_params=False, conv_w=None, conv_b=None,
            zoh=False, threads=0):
    """Routed forward pass in fp64.

    Shapes: u, delta [b, tokens, D] (or [K, b, tokens, D] with per_dir_inputs);
    B, C [b, tokens, N] (or [K, ...]); A [D, N] (or [K, D, N] with per_dir_params);
    Dskip, bias [D] (or [K, D]); z [b, tokens, D]. Returns y [b, tokens, D] float64.
    conv_w [D, 4] (or [K, D, 4]) and conv_b [D] (or [K, D]) fuse the causal
    kernel-four convolution + SiLU into u (BIDIR and pooled routes only);
    zoh=True uses the zero-order-hold write term.
    """
    K, L, T = geometry(kind, h, w, cls_pos)
    u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
    Dskip = None if Dskip is None else _f64(Dskip)
    bias = None if bias is None else _f64(bias)
    z = None if z is None else _f64(z)
    lead = 1 if per_dir_inputs else 0
    if per_dir_inputs:
        assert u.shape[0] == K and delta.shape[0] == K and B.shape[0] == K and C.shape[0] == K
    b, tok, D = u.shape[lead:]
    N = B.shape[-1]
    assert tok == T, f"token count {tok} != route tokens {T}"
    assert delta.shape == u.shape and C.shape == B.shape
    assert B.shape[lead:] == (b, T, N)
    assert A.shape[-2:] == (D, N)
    if per_dir_params:
        assert A.shape[0] == K
    if z is not None:
        assert z.shape == (b, T, D)
    conv_w = None if conv_w is None else _f64(conv_w)
    conv_b = None if conv_b is None else _f64(conv_b)
    if conv_w is not None:
        assert conv_w.shape == ((K, D, 4) if per_dir_params else (D, 4))
        if conv_b is not None:
            assert conv_b.shape == ((K, D) if per_dir_params else (D,))
    y = np.empty((b, T, D), dtype=np.float64)
    rc = _load().oracle_forward(_kind(kind), h, w, cls_pos, b, D, N, _ptr(u), _ptr(delta),
                                _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(bias), _ptr(z),
                                int(bool(delta_softplus)), float(merge_scale),
                                int(bool(per_dir_inputs)), int(bool(per_dir_params)),
                                _ptr(conv_w), _ptr(conv_b), int(bool(zoh)),
                                _ptr(y), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_forward failed (rc={rc})")
    return y


def forward_masked(kind, h, w, pos, u, delta, A, B, C, Dskip=None, bias=None, z=None, *,
                   delta_softplus=True, merge_scale=1.0, per_dir_inputs=False,
                   per_dir_params=False, zoh=False, threads=0):
    """Pooled route on a masked token set (FastMaskVim) in fp64.

    pos [b, n] int grid positions (row * w + col) of the visible tokens; u, delta
    [b, n, D] (or [2, b, n, D]); B, C [b, n, N] (or [2, ...]); z [b, n, D].
    Pooled tokens are row (POOL_W) or column (POOL_H) sums over the visible
    tokens divided by the nominal width (height). Returns y [b, n, D].
    """
    u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int32))
    Dskip = None if Dskip is None else _f64(Dskip)
    bias = None if bias is None else _f64(bias)
    z = None if z is None else _f64(z)
    lead = 1 if per_dir_inputs else 0
    b, n, D = u.shape[lead:]
    N = B.shape[-1]
    assert pos.shape == (b, n) and delta.shape == u.shape and C.shape == B.shape
    y = np.empty((b, n, D), dtype=np.float64)
    rc = _load().oracle_forward_masked(_kind(kind), h, w, b, n, _ptr(pos), D, N, _ptr(u), _ptr(delta),
                                       _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip), _ptr(bias), _ptr(z),
                                       int(bool(delta_softplus)), float(merge_scale),
                                       int(bool(per_dir_inputs)), int(bool(per_dir_params)),
                                       int(bool(zoh)), _ptr(y), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_forward_masked failed (rc={rc})")
    return y


def backward(kind, h, w, u, delta, A, B, C, Dskip=None, bias=None, z=None, *, dy, cls_pos=-1,
             delta_softplus=True, merge_scale=1.0, per_dir_inputs=False, per_dir_params=False,
             threads=0):
    """Gradients of forward() w.r.t. every input, given dy = dL/dy, in fp64.

    Returns a dict: du, ddelta (w.r.t. the raw step), dB, dC (shapes of the inputs),
    dA, dDskip, dbias (shapes of the parameters) and dz (when z is given).
    """
    K, L, T = geometry(kind, h, w, cls_pos)
    u, delta, A, B, C, dy = map(_f64, (u, delta, A, B, C, dy))
    Dskip = None if Dskip is None else _f64(Dskip)
    bias = None if bias is None else _f64(bias)
    z = None if z is None else _f64(z)
    lead = 1 if per_dir_inputs else 0
    b, tok, D = u.shape[lead:]
    N = B.shape[-1]
    assert tok == T and dy.shape == (b, T, D)
    Kp = K if per_dir_params else 1
    out = dict(du=np.empty(u.shape), ddelta=np.empty(u.shape), dB=np.empty(B.shape), dC=np.empty(C.shape),
               dA=np.empty(A.shape), dDskip=np.empty((Kp, D) if per_dir_params else (D,)),
               dbias=np.empty((Kp, D) if per_dir_params else (D,)))
    if z is not None:
        out["dz"] = np.empty(z.shape)
    rc = _load().oracle_backward(_kind(kind), h, w, cls_pos, b, D, N, _ptr(u), _ptr(delta), _ptr(A),
                                 _ptr(B), _ptr(C), _ptr(Dskip), _ptr(bias), _ptr(z),
                                 int(bool(delta_softplus)), float(merge_scale), int(bool(per_dir_inputs)),
                                 int(bool(per_dir_params)), _ptr(dy), _ptr(out["du"]), _ptr(out["ddelta"]),
                                 _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dDskip"]),
                                 _ptr(out["dbias"]), _ptr(out.get("dz")), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_backward failed (rc={rc})")
    return out
