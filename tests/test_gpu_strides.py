"""Strided tensors (vscan_args token and image strides) on the GPU.

u, delta, z and y are views of wider buffers (padding after every token row and
after every image), B and C likewise with their own strides; per-direction
inputs are views of [K, batch, T', D'] buffers. The library packs the views
into its workspace, runs the dense path and copies y out, so the result must
equal the dense call bit for bit, match the fp64 oracle, and leave every
element of the output buffer outside the view untouched.
"""
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import workloads
from vscan_testlib import TOL, rel_err, run_oracle, small_workload, to_device

import vision_selective_state_b200 as vs

pytestmark = pytest.mark.gpu

SENTINEL = 7.25


def _view(t, pad_rows, pad_tok):
    """A view of t ([(K,) batch, T, R]) inside a buffer with pad_rows more elements per
    row and pad_tok more token rows per image, filled with SENTINEL around the view."""
    shape = list(t.shape)
    big = torch.full(shape[:-2] + [shape[-2] + pad_tok, shape[-1] + pad_rows], SENTINEL, dtype=t.dtype,
                     device=t.device)
    v = big[..., : shape[-2], : shape[-1]]
    v.copy_(t)
    return big, v


@pytest.mark.parametrize("route,h,w", [("bidir", 8, 8), ("cross4", 6, 7), ("atrous2", 5, 7), ("pool_w", 8, 8),
                                       ("pool_h", 6, 9)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("pad_rows,pad_tok,pad_bc", [(8, 0, 0), (0, 3, 0), (16, 2, 5), (0, 0, 3)])
def test_strided_views_match_the_dense_call(route, h, w, dtype, pad_rows, pad_tok, pad_bc):
    D, N, batch = 24, 16, 3
    wl = small_workload(route, h, w, D, N, dtype, batch, seed=11)
    x = workloads.draw(wl, a_mode="random")
    r = vs.Route(route, h, w, wl.cls_pos)
    xd = to_device(x, dtype)
    dense = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"])
    _, u = _view(xd["u"], pad_rows, pad_tok)
    _, dl = _view(xd["delta"], pad_rows, pad_tok)
    _, z = _view(xd["z"], pad_rows, pad_tok)
    ybig, y = _view(torch.zeros_like(xd["z"]), pad_rows, pad_tok)
    ybig.fill_(SENTINEL)
    _, B = _view(xd["B"], pad_bc, pad_tok)
    _, C = _view(xd["C"], pad_bc, pad_tok)
    assert not u.is_contiguous() or not B.is_contiguous()
    out = vs.forward(r, u, dl, xd["A"], B, C, xd["Dskip"], xd["bias"], z, out=y)
    torch.cuda.synchronize()
    assert out.data_ptr() == y.data_ptr()
    assert torch.equal(y, dense), (route, dtype)
    # nothing written outside the view
    mask = torch.ones_like(ybig, dtype=torch.bool)
    mask[..., : y.shape[-2], : y.shape[-1]] = False
    assert bool((ybig[mask] == SENTINEL).all())
    ref = run_oracle(route, h, w, wl.cls_pos, x)
    assert rel_err(y.float().cpu().numpy(), ref) <= TOL[dtype]


@pytest.mark.parametrize("route,h,w", [("bidir", 7, 9), ("cross4", 5, 6)])
def test_strided_per_direction_planes(route, h, w):
    D, N, batch, dtype = 16, 16, 2, "bf16"
    wl = small_workload(route, h, w, D, N, dtype, batch, seed=5)
    x = workloads.draw(wl, a_mode="random", per_dir_inputs=True, per_dir_params=True)
    r = vs.Route(route, h, w, wl.cls_pos)
    xd = to_device(x, dtype)
    kw = dict(per_dir_inputs=True, per_dir_params=True)
    dense = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"], **kw)
    _, u = _view(xd["u"], 8, 2)
    _, dl = _view(xd["delta"], 8, 2)
    _, z = _view(xd["z"], 8, 2)
    _, B = _view(xd["B"], 4, 2)
    _, C = _view(xd["C"], 4, 2)
    y = vs.forward(r, u, dl, xd["A"], B, C, xd["Dskip"], xd["bias"], z, **kw)  # y allocated in u's layout
    torch.cuda.synchronize()
    assert y.stride() == z.stride()
    assert torch.equal(y, dense)
    ref = run_oracle(route, h, w, wl.cls_pos, x, **kw)
    assert rel_err(y.float().cpu().numpy(), ref) <= TOL[dtype]


def test_strided_call_with_value_checks_and_no_gate():
    route, h, w, D, N, batch, dtype = "bidir", 6, 6, 16, 16, 2, "f32"
    wl = small_workload(route, h, w, D, N, dtype, batch, seed=9)
    x = workloads.draw(wl, a_mode="random")
    r = vs.Route(route, h, w, wl.cls_pos)
    xd = to_device(x, dtype)
    dense = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], None)
    _, u = _view(xd["u"], 4, 1)
    _, dl = _view(xd["delta"], 4, 1)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = vs.forward(r, u, dl, xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], None, status=status,
                   check_values=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(y, dense)
    u[0, 0, 0] = float("nan")  # a non-finite value inside the view is found in the packed copy
    vs.forward(r, u, dl, xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], None, status=status, check_values=True)
    torch.cuda.synchronize()
    assert vs.status_from_device_word(int(status.item())) == -7
