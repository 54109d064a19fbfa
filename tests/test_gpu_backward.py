"""CUDA backward pass vs the fp64 oracle's backward (itself pinned by finite
differences): every gradient, every route, sequences spanning several 16-step
chunks with ragged tails, per-direction inputs and parameters, the optional
terms, and both I/O types. Gradients are float32 and summed with atomics, so
they are compared with the tolerance metric, not bit for bit.
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

KEYS = ("du", "ddelta", "dB", "dC", "dA", "dDskip", "dbias", "dz")


def _case(route, h, w, D, dtype, *, N=16, batch=2, seed=11, pdi=False, pdp=False, gate=True, skip=True,
          bias=True, softplus=True, merge_scale=0.7, cls=None):
    wl = small_workload(route, h, w, D, N, dtype, batch, seed, cls)
    x = workloads.draw(wl, a_mode="random", per_dir_inputs=pdi, per_dir_params=pdp)
    if not softplus:
        x["delta"] = np.abs(x["delta"])
        x["bias"] = np.full_like(x["bias"], 0.01)
    rng = np.random.default_rng(seed + 3)
    dy = rng.standard_normal((batch, wl.tokens, D)).astype(np.float32)
    if dtype == "bf16":
        dy = workloads.round_to_bf16(dy)
    xd = to_device(x, dtype)
    dyd = torch.from_numpy(dy).to("cuda", torch.bfloat16 if dtype == "bf16" else torch.float32)
    r = vs.Route(route, h, w, wl.cls_pos)
    g = vs.backward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"] if skip else None,
                    xd["bias"] if bias else None, xd["z"] if gate else None, dy=dyd, delta_softplus=softplus,
                    merge_scale=merge_scale, per_dir_inputs=pdi, per_dir_params=pdp)
    torch.cuda.synchronize()
    ref = O.backward(route, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"] if skip else None,
                     x["bias"] if bias else None, x["z"] if gate else None, dy=dy, cls_pos=wl.cls_pos,
                     delta_softplus=softplus, merge_scale=merge_scale, per_dir_inputs=pdi, per_dir_params=pdp)
    tol = TOL[dtype]
    for k in KEYS:
        if k not in ref or k not in g:
            continue
        err = rel_err(g[k].cpu().numpy(), ref[k])
        assert err <= tol, (route, h, w, dtype, k, err)


@pytest.mark.parametrize("route", ["bidir", "cross4", "atrous2", "pool_w", "pool_h"])
@pytest.mark.parametrize("h,w", [(1, 1), (3, 5), (9, 13), (17, 19)])
def test_backward_f32(route, h, w):
    _case(route, h, w, 24, "f32")


@pytest.mark.parametrize("route", ["bidir", "cross4", "atrous2", "pool_w"])
def test_backward_bf16(route):
    _case(route, 11, 14, 16, "bf16")


@pytest.mark.parametrize("route", ["bidir", "cross4", "atrous2", "pool_w", "pool_h"])
def test_backward_per_direction(route):
    _case(route, 7, 9, 16, "f32", pdi=True, pdp=True)


@pytest.mark.parametrize("route", ["bidir", "atrous2", "pool_h"])
def test_backward_without_optional_terms_and_state_tail(route):
    _case(route, 6, 7, 12, "f32", N=5, gate=False, skip=False, bias=False, softplus=False, merge_scale=1.0)


def test_backward_bidir_with_middle_cls_and_long_sequence():
    _case("bidir", 14, 14, 16, "f32", cls=98)
    _case("bidir", 31, 33, 8, "f32", batch=1)


@pytest.mark.parametrize("route,h,w,D,dtype,batch,kw", [
    ("bidir", 5, 7, 196, "f32", 64, {}),                          # 25 tiles (channel tail) x 64 x 2
    ("bidir", 6, 6, 64, "bf16", 96, {"pdi": True}),               # 8 x 96 x 2
    ("bidir", 4, 6, 24, "f32", 256, {"gate": False, "skip": False, "bias": False, "softplus": False,
                                     "merge_scale": 1.0}),       # 3 x 256 x 2
    ("cross4", 5, 6, 64, "bf16", 96, {"N": 7}),                   # 8 x 96 x 4, plain loads
    ("cross4", 5, 6, 64, "bf16", 48, {}),                         # 8 x 48 x 4
    ("cross4", 5, 5, 24, "f32", 128, {"N": 7, "pdi": True, "pdp": True}),  # 3 x 128 x 4
    ("atrous2", 5, 7, 24, "f32", 160, {"pdi": True, "pdp": True}),  # 3 x 160 x 4
    ("atrous2", 7, 5, 16, "bf16", 192, {}),                       # 2 x 192 x 4
    ("pool_w", 6, 9, 104, "f32", 96, {}),                         # 13 x 96 x 2 over the pooled sequence
    ("pool_h", 5, 8, 48, "bf16", 128, {"N": 5, "pdp": True}),     # 6 x 128 x 2, plain loads
])
def test_backward_large_grids_take_the_one_warp_register_capped_build(route, h, w, D, dtype, batch, kw):
    """Grids of more than 8 tiles per SM (here 1536-3200 tiles) run the adjoint scan with
    one warp per tile, built for 16 resident warps per SM, which sums dB and dC with a
    per-step shuffle reduce-scatter; the pooled routes also run its forward pass (no
    saved checkpoints). Smaller grids, every other case in this file, run the build that
    splits a tile's states over two warps."""
    _case(route, h, w, D, dtype, batch=batch, **kw)


def test_backward_refuses_unsupported_options():
    r = vs.Route("bidir", 4, 4)
    x = torch.zeros(1, 16, 8, device="cuda")
    bc = torch.zeros(1, 16, 16, device="cuda")
    A = -torch.ones(8, 16, device="cuda")
    import ctypes
    from vision_selective_state_b200 import _abi
    a = vs._args(r, x, x, A, bc, bc, None, None, None, x, True, 1.0, False, False, None, 0, None, None, True)
    n = ctypes.c_uint64()
    assert _abi.lib.vscan_backward_workspace_size(r.handle, ctypes.byref(a), ctypes.byref(n)) == -4
