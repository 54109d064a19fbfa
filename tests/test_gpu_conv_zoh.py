"""CUDA path vs the fp64 oracle for the two optional steps: the fused causal
convolution (+ SiLU) of u and the zero-order-hold write term.

Convolution: BIDIR through both the streaming kernel (steps read across 16-step
chunk boundaries) and the resident chunked kernel, with and without CLS,
shared and per-direction kernels; the pooled routes with the convolution
running along the row-major / column-major sequence across grid rows, shared
and per-direction inputs. ZOH: every route and kernel. Both I/O types, ragged
channel tiles and sequence tails, and both steps together.
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


def _case(route, h, w, D, dtype, *, conv=False, zoh=False, batch=2, seed=3, pdi=False, pdp=False,
          cls=None, seq_chunks=0, N=16, a_mode="random", host=False):
    wl = small_workload(route, h, w, D, N, dtype, batch, seed, cls)
    x = workloads.draw(wl, a_mode=a_mode, per_dir_inputs=pdi, per_dir_params=pdp)
    cv = workloads.draw_conv(wl, per_dir_params=pdp) if conv else dict(conv_w=None, conv_b=None)
    r = vs.Route(route, h, w, wl.cls_pos)
    cw = None if cv["conv_w"] is None else torch.from_numpy(cv["conv_w"])
    cb = None if cv["conv_b"] is None else torch.from_numpy(cv["conv_b"])
    if host:
        xh = to_device(x, dtype, device="cpu")
        out = torch.empty(xh["z"].shape, dtype=xh["u"].dtype).pin_memory()
        nbytes = vs.host_buffer_size(r, xh["u"], xh["B"], per_dir_inputs=pdi, per_dir_params=pdp,
                                     conv_w=conv, conv_b=conv)
        buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        vs.forward_host(r, xh["u"], xh["delta"], xh["A"], xh["B"], xh["C"], xh["Dskip"], xh["bias"],
                        xh["z"], out=out, device_buffer=buf, per_dir_inputs=pdi, per_dir_params=pdp,
                        conv_w=cw, conv_b=cb, zoh=zoh)
        torch.cuda.synchronize()
        y = out
    else:
        xd = to_device(x, dtype)
        y = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"],
                       xd["z"], per_dir_inputs=pdi, per_dir_params=pdp, seq_chunks=seq_chunks,
                       conv_w=None if cw is None else cw.cuda(), conv_b=None if cb is None else cb.cuda(),
                       zoh=zoh)
        torch.cuda.synchronize()
    ref = O.forward(route, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"],
                    x["z"], cls_pos=wl.cls_pos, per_dir_inputs=pdi, per_dir_params=pdp,
                    conv_w=cv["conv_w"], conv_b=cv["conv_b"], zoh=zoh)
    err = rel_err(y.float().cpu().numpy(), ref)
    assert err <= TOL[dtype], (route, h, w, D, dtype, conv, zoh, seq_chunks, err)
    return err


# ------------------------------------------------------------------- convolution
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("h,w,cls", [(1, 1, -1), (1, 5, 2), (3, 5, 7), (9, 13, 58), (31, 33, -1)])
@pytest.mark.parametrize("seq_chunks", [1, 0])
def test_conv_bidir(dtype, h, w, cls, seq_chunks):
    D = 40 if dtype == "f32" else 24
    _case("bidir", h, w, D, dtype, conv=True, cls=cls, seq_chunks=seq_chunks)


@pytest.mark.parametrize("seq_chunks", [2, 4, 8])
@pytest.mark.parametrize("pdp,pdi", [(False, False), (True, False), (True, True)])
def test_conv_bidir_resident_and_per_direction(seq_chunks, pdp, pdi):
    _case("bidir", 14, 14, 24, "f32", conv=True, cls=98, seq_chunks=seq_chunks, pdp=pdp, pdi=pdi)


@pytest.mark.parametrize("pdp,pdi", [(True, False), (True, True)])
def test_conv_bidir_streaming_per_direction(pdp, pdi):
    _case("bidir", 19, 21, 16, "f32", conv=True, seq_chunks=1, pdp=pdp, pdi=pdi)


@pytest.mark.parametrize("route", ["pool_w", "pool_h"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("h,w", [(1, 1), (5, 1), (1, 7), (16, 24), (33, 17)])
def test_conv_pooled(route, dtype, h, w):
    D = 40 if dtype == "f32" else 48
    _case(route, h, w, D, dtype, conv=True)


@pytest.mark.parametrize("route", ["pool_w", "pool_h"])
@pytest.mark.parametrize("pdp,pdi", [(True, False), (False, True), (True, True)])
def test_conv_pooled_per_direction(route, pdp, pdi):
    _case(route, 12, 10, 36, "f32", conv=True, pdp=pdp, pdi=pdi)


@pytest.mark.parametrize("route", ["cross4", "atrous2"])
def test_conv_is_unsupported_on_grid_routes(route):
    r = vs.Route(route, 4, 4)
    x = torch.zeros(1, 16, 8, device="cuda")
    bc = torch.zeros(1, 16, 16, device="cuda")
    A = -torch.ones(8, 16, device="cuda")
    with pytest.raises(vs.VscanError):
        vs.forward(r, x, x, A, bc, bc, conv_w=torch.zeros(8, 4, device="cuda"))


# ------------------------------------------------------------------ zero-order hold
@pytest.mark.parametrize("route", ["bidir", "cross4", "atrous2", "pool_w", "pool_h"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("h,w", [(1, 1), (6, 4), (13, 11), (17, 19)])
def test_zoh_all_routes(route, dtype, h, w):
    D = 24 if dtype == "f32" else 16
    _case(route, h, w, D, dtype, zoh=True, seq_chunks=1 if route in ("cross4", "atrous2", "bidir") else 0)


@pytest.mark.parametrize("batch", [2, 40])
def test_zoh_atrous_f32_both_consumer_layouts(batch):
    """The ZOH write term on the float32 atrous streaming kernel with the states split
    over two consumer warps (at most 8 CTAs per SM) and with one consumer warp (1280
    CTAs)."""
    _case("atrous2", 5, 7, 64, "f32", zoh=True, batch=batch, seq_chunks=1)


@pytest.mark.parametrize("zoh,conv", [(True, False), (False, True), (True, True)])
def test_resident_wide_tile_with_optional_steps(zoh, conv):
    """The 8-channel BIDIR resident tile (1188 channels, 149 tiles at batch 1) with the
    zero-order-hold term and the fused convolution."""
    _case("bidir", 7, 6, 1188, "f32", zoh=zoh, conv=conv, batch=1, seq_chunks=8)
    _case("bidir", 7, 6, 1188, "f32", zoh=zoh, conv=conv, batch=2, seq_chunks=4, pdi=True, pdp=True)


@pytest.mark.parametrize("route", ["bidir", "cross4", "atrous2"])
@pytest.mark.parametrize("seq_chunks", [2, 8])
def test_zoh_resident(route, seq_chunks):
    _case(route, 9, 13, 16, "f32", zoh=True, seq_chunks=seq_chunks)


@pytest.mark.parametrize("route", ["bidir", "pool_w"])
@pytest.mark.parametrize("N", [16, 5])
def test_zoh_with_s4d_decays_and_state_tails(route, N):
    _case(route, 10, 12, 20, "f32", zoh=True, N=N, a_mode="s4d")


# ----------------------------------------------------------------------- together
@pytest.mark.parametrize("route,seq_chunks", [("bidir", 1), ("bidir", 4), ("pool_w", 0), ("pool_h", 0)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_and_zoh_together(route, seq_chunks, dtype):
    _case(route, 11, 14, 16 if dtype == "bf16" else 20, dtype, conv=True, zoh=True, seq_chunks=seq_chunks,
          cls=-1)


@pytest.mark.parametrize("route", ["bidir", "pool_w"])
def test_conv_and_zoh_through_host_buffers(route):
    _case(route, 8, 9, 16, "f32", conv=True, zoh=True, host=True, cls=-1)
