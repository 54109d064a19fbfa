"""CUDA path vs the fp64 oracle on masked token sets (FastMaskVim: the pooled
routes over visible tokens addressed by grid position, row sums normalized by
the nominal width).

Random per-image masks at MAE-like keep ratios, both pooled axes and I/O types,
per-direction inputs and parameters, the zero-order-hold term, the host-buffer
and the no-allocation entry points, an empty token set, and positions outside
the grid (skipped; their y is 0).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import oracle as O
import workloads
from vscan_testlib import TOL, rel_err, small_workload, to_device

import vision_selective_state_b200 as vs

pytestmark = pytest.mark.gpu


def _masked_inputs(route, h, w, D, dtype, keep, batch, seed, pdi=False, pdp=False, N=16):
    wl = small_workload(route, h, w, D, N, dtype, batch, seed)
    n = max(1, int(round(keep * h * w)))
    x = workloads.draw(wl.with_(h=n, w=1), per_dir_inputs=pdi, per_dir_params=pdp, a_mode="random")
    r = np.random.default_rng(seed + 1)
    pos = np.stack([np.sort(r.choice(h * w, n, replace=False)) for _ in range(batch)]).astype(np.int32)
    return wl, x, pos


def _run(route, h, w, x, pos, dtype, pdi=False, pdp=False, zoh=False, host=False, noalloc=False):
    r = vs.Route(route, h, w)
    if host:
        xh = to_device(x, dtype, device="cpu")
        out = torch.empty(xh["z"].shape, dtype=xh["u"].dtype).pin_memory()
        tp = torch.from_numpy(pos)
        nbytes = vs.host_buffer_size(r, xh["u"], xh["B"], per_dir_inputs=pdi, per_dir_params=pdp,
                                     token_pos=True)
        buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        vs.forward_host(r, xh["u"], xh["delta"], xh["A"], xh["B"], xh["C"], xh["Dskip"], xh["bias"], xh["z"],
                        out=out, device_buffer=buf, per_dir_inputs=pdi, per_dir_params=pdp, zoh=zoh,
                        token_pos=tp)
        torch.cuda.synchronize()
        return out.float().numpy()
    xd = to_device(x, dtype)
    tp = torch.from_numpy(pos).cuda()
    if noalloc:
        import ctypes
        from vision_selective_state_b200 import _abi
        y = torch.empty_like(xd["z"])
        a = vs._args(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"], y,
                     True, 1.0, pdi, pdp, None, 0, None, None, zoh, tp)
        _abi.check(_abi.lib.vscan_forward_pooled_noalloc(r.handle, ctypes.byref(a),
                                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))
    else:
        y = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
                       per_dir_inputs=pdi, per_dir_params=pdp, zoh=zoh, token_pos=tp)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


def _check(route, h, w, D, dtype, keep, *, batch=3, seed=5, pdi=False, pdp=False, zoh=False, host=False,
           noalloc=False, N=16):
    wl, x, pos = _masked_inputs(route, h, w, D, dtype, keep, batch, seed, pdi, pdp, N)
    y = _run(route, h, w, x, pos, dtype, pdi, pdp, zoh, host, noalloc)
    ref = O.forward_masked(route, h, w, pos, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"],
                           x["bias"], x["z"], per_dir_inputs=pdi, per_dir_params=pdp, zoh=zoh)
    err = rel_err(y, ref)
    assert err <= TOL[dtype], (route, h, w, keep, dtype, err)


@pytest.mark.parametrize("route", ["pool_w", "pool_h"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("h,w,keep", [(1, 1, 1.0), (8, 1, 0.5), (16, 24, 0.25), (33, 17, 0.25),
                                      (20, 20, 1.0), (64, 48, 0.1)])
def test_masked_pooled(route, dtype, h, w, keep):
    _check(route, h, w, 40 if dtype == "f32" else 48, dtype, keep)


@pytest.mark.parametrize("route", ["pool_w", "pool_h"])
@pytest.mark.parametrize("pdi,pdp", [(True, False), (False, True), (True, True)])
def test_masked_per_direction(route, pdi, pdp):
    _check(route, 12, 14, 24, "f32", 0.3, pdi=pdi, pdp=pdp)


@pytest.mark.parametrize("route", ["pool_w", "pool_h"])
def test_masked_zoh_state_tail_and_entry_points(route):
    _check(route, 15, 11, 16, "f32", 0.4, zoh=True, N=7)
    _check(route, 15, 11, 16, "f32", 0.4, host=True)
    _check(route, 15, 11, 16, "f32", 0.4, noalloc=True)


def test_positions_outside_the_grid_are_skipped_and_zeroed():
    h, w, D = 6, 7, 8
    wl, x, pos = _masked_inputs("pool_w", h, w, D, "f32", 0.5, 2, 9)
    bad = pos.copy()
    bad[0, 3], bad[1, 0] = -1, h * w  # two tokens outside the grid
    y = _run("pool_w", h, w, x, bad, "f32")
    assert np.all(y[0, 3] == 0) and np.all(y[1, 0] == 0)
    for i, drop in ((0, 3), (1, 0)):
        keep = [t for t in range(pos.shape[1]) if t != drop]
        sub = {k: (v[i:i + 1, keep] if k in ("u", "delta", "B", "C", "z") else v) for k, v in x.items()}
        ref = O.forward_masked("pool_w", h, w, bad[i:i + 1, keep], sub["u"], sub["delta"], sub["A"], sub["B"],
                               sub["C"], sub["Dskip"], sub["bias"], sub["z"])
        assert rel_err(y[i:i + 1, keep], ref) <= TOL["f32"]


def test_empty_token_set():
    r = vs.Route("pool_w", 4, 4)
    u = torch.zeros(2, 0, 8, device="cuda")
    bc = torch.zeros(2, 0, 16, device="cuda")
    y = vs.forward(r, u, u, -torch.ones(8, 16, device="cuda"), bc, bc,
                   token_pos=torch.zeros(2, 0, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert y.shape == (2, 0, 8)
