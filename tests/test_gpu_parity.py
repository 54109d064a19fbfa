"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small cases span several 16-step chunks and 8-channel tiles with ragged tails,
degenerate grids (1x1, single rows and columns), every route, both I/O types,
N != 16, per-direction inputs and parameters, and the optional terms. Full-size
workloads run in the launch configuration the benchmark times and are checked
on sampled images and channels (channels and images are independent, so the
oracle computes those exactly).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import oracle as O
import workloads
from vscan_testlib import TOL, rel_err, run_gpu, run_oracle, small_workload, to_device

import vision_selective_state_b200 as vs

pytestmark = pytest.mark.gpu

ROUTES = ["bidir", "cross4", "atrous2", "pool_w", "pool_h"]


def _case(route, h, w, D, N, dtype, batch=2, seed=1, a_mode="random", pdi=False, pdp=False, cls=None, **opts):
    wl = small_workload(route, h, w, D, N, dtype, batch, seed, cls)
    x = workloads.draw(wl, a_mode=a_mode, per_dir_inputs=pdi, per_dir_params=pdp)
    if opts.get("delta_softplus") is False:
        # without softplus the step is raw delta + bias: keep it positive (stable decay)
        x["delta"] = np.abs(x["delta"])
        x["bias"] = np.full_like(x["bias"], 0.01)
    r = vs.Route(route, h, w, wl.cls_pos)
    y = run_gpu(r, to_device(x, dtype), per_dir_inputs=pdi, per_dir_params=pdp, **opts)
    opts.pop("seq_chunks", None)  # a launch choice of the CUDA path only
    ref = run_oracle(route, h, w, wl.cls_pos, x, per_dir_inputs=pdi, per_dir_params=pdp, **opts)
    err = rel_err(y.float().cpu().numpy(), ref)
    assert err <= TOL[dtype], (route, h, w, D, N, dtype, err)
    return err


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("h,w", [(1, 1), (1, 9), (9, 1), (3, 5), (6, 4), (13, 11), (16, 17)])
def test_small_grids(route, dtype, h, w):
    D = 24 if dtype == "f32" else 16
    _case(route, h, w, D, 16, dtype)


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("D,N", [(4, 1), (12, 3), (20, 16), (36, 7), (8, 12)])
def test_channel_and_state_tails(route, D, N):
    _case(route, 7, 10, D, N, "f32")


@pytest.mark.parametrize("route", ROUTES)
def test_per_direction_inputs_and_parameters(route):
    _case(route, 9, 7, 16, 16, "f32", pdi=True, pdp=True)
    _case(route, 9, 7, 16, 16, "bf16", pdi=False, pdp=True)
    _case(route, 9, 7, 16, 16, "f32", pdi=True, pdp=False)


@pytest.mark.parametrize("route", ROUTES)
def test_optional_terms(route):
    _case(route, 8, 9, 16, 16, "f32", gate=False)
    _case(route, 8, 9, 16, 16, "f32", skip=False, bias=False)
    _case(route, 8, 9, 16, 16, "f32", merge_scale=0.5)
    _case(route, 8, 9, 16, 16, "f32", delta_softplus=False, a_mode="s4d")


@pytest.mark.parametrize("route", ["bidir", "cross4", "atrous2"])
@pytest.mark.parametrize("nc", [1, 2, 4, 8])
@pytest.mark.parametrize("h,w", [(1, 1), (3, 5), (14, 14), (9, 13)])
def test_resident_chunked_scan(route, nc, h, w):
    """The chunked parallel scan (affine-pair prefix over chunks) against the oracle,
    with chunk boundaries falling on every kind of step (pads, CLS, ragged ends)."""
    _case(route, h, w, 12, 16, "f32", seq_chunks=nc)
    _case(route, h, w, 16, 7, "bf16", seq_chunks=nc, pdi=True, pdp=True)
    _case(route, h, w, 8, 16, "f32", seq_chunks=nc, merge_scale=0.5, gate=False)


@pytest.mark.parametrize("batch,D", [(2, 24), (40, 64)])
def test_atrous_f32_streaming_consumer_layouts(batch, D):
    """float32 atrous streaming launches of at most 4 CTAs per SM (2 x 3 x 4 = 24 here)
    split each channel's 16 states over two consumer warps; larger ones (40 x 8 x 4 =
    1280) keep one consumer warp per 8 channels. Both against the oracle, with a
    ragged channel tile, per-direction planes and the options."""
    _case("atrous2", 5, 7, D, 16, "f32", batch=batch, seq_chunks=1)
    _case("atrous2", 7, 6, D, 16, "f32", batch=batch, seq_chunks=1, pdi=True, pdp=True)
    _case("atrous2", 5, 7, D, 7, "f32", batch=batch, seq_chunks=1, gate=False, merge_scale=0.5)


@pytest.mark.parametrize("nc", [2, 4, 8])
def test_resident_tile_widths(nc):
    """BIDIR resident tiles are 4 channels wide while 8-channel tiles would leave SMs
    without a CTA, else 8: 1188 channels (149 eight-channel tiles, the last one half
    past the end) at batch 1 and 2 take the wide tile, 384 channels at batch 1 the
    narrow one; f32 with N = 16 stages by cp.async pieces, the others element-wise."""
    _case("bidir", 5, 6, 1188, 16, "f32", batch=1, seq_chunks=nc)
    _case("bidir", 5, 6, 1188, 16, "f32", batch=2, seq_chunks=nc, pdi=True, pdp=True)
    _case("bidir", 5, 6, 1188, 16, "f32", batch=1, seq_chunks=nc, gate=False)
    _case("bidir", 5, 6, 1192, 7, "bf16", batch=1, seq_chunks=nc, pdp=True)
    _case("bidir", 6, 5, 1192, 16, "bf16", batch=1, seq_chunks=nc)
    _case("bidir", 14, 14, 384, 16, "f32", batch=1, seq_chunks=nc, pdp=True)


@pytest.mark.parametrize("route,h,w", [("bidir", 14, 14), ("cross4", 9, 13), ("atrous2", 9, 13),
                                       ("bidir", 31, 33), ("cross4", 31, 33), ("atrous2", 31, 33)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_streaming_kernel_full_state_rows(route, h, w, dtype):
    """The streaming kernel (seq_chunks=1) with N = 16, both I/O types, short and long sequences."""
    _case(route, h, w, 16, 16, dtype, seq_chunks=1)


def test_bidirectional_without_cls_and_long_sequences():
    _case("bidir", 10, 10, 16, 16, "f32", cls=-1)
    _case("bidir", 40, 40, 16, 16, "f32", batch=1)       # L = 1601, CLS 800
    _case("cross4", 31, 33, 8, 16, "bf16", batch=1)      # L = 1023


@pytest.mark.parametrize("h,w,cls", [(45, 46, 1035), (32, 64, -1), (47, 47, 1104)])
def test_bidirectional_long_bf16_sequences_use_32_step_chunks(h, w, cls):
    """bf16 BIDIR sequences of 2048 steps or more stream in 32-step chunks: ragged
    last chunks (L = 2071, 2210) and an exact multiple (L = 2048, no CLS); N = 16 and
    N < 16; shared and per-direction inputs; a channel tail (24 = 8-channel tiles x 3)."""
    _case("bidir", h, w, 16, 16, "bf16", batch=1, cls=cls, seq_chunks=1)
    _case("bidir", h, w, 24, 7, "bf16", batch=1, cls=cls, seq_chunks=1, pdi=True, pdp=True)


def test_empty_batch_is_a_no_op():
    r = vs.Route("atrous2", 4, 4)
    wl = small_workload("atrous2", 4, 4, 8, 16, "f32", 1, 3)
    xd = to_device(workloads.draw(wl), "f32")
    e = {k: (v[:0] if k in ("u", "delta", "B", "C", "z") else v) for k, v in xd.items()}
    y = vs.forward(r, e["u"], e["delta"], e["A"], e["B"], e["C"], e["Dskip"], e["bias"], e["z"])
    torch.cuda.synchronize()
    assert y.shape == (0, 16, 8)


@pytest.mark.parametrize("kind,h,w", [("bidir", 14, 14), ("bidir", 1, 1), ("cross4", 7, 5),
                                      ("atrous2", 3, 5), ("atrous2", 55, 57), ("atrous2", 1, 1),
                                      ("pool_w", 5, 9), ("pool_h", 5, 9), ("cross4", 56, 56)])
def test_route_maps_are_bit_exact(kind, h, w):
    cls = (h * w) // 2 if kind == "bidir" else -1
    r = vs.Route(kind, h, w, cls)
    got = r.indices().cpu().numpy().astype(np.int64)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got, O.route(kind, h, w, cls))


def test_host_buffer_path_matches_device_path():
    wl = small_workload("cross4", 12, 10, 16, 16, "bf16", 2, 5)
    x = workloads.draw(wl)
    r = vs.Route("cross4", 12, 10)
    xd = to_device(x, "bf16")
    y_dev = run_gpu(r, xd).cpu()
    xh = {k: v.cpu().pin_memory() for k, v in xd.items()}
    out = torch.empty_like(xh["u"]).pin_memory()
    nbytes = vs.host_buffer_size(r, xh["u"], xh["B"])
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    vs.forward_host(r, xh["u"], xh["delta"], xh["A"], xh["B"], xh["C"], xh["Dskip"], xh["bias"],
                    xh["z"], out=out, device_buffer=buf)
    torch.cuda.synchronize()
    assert torch.equal(out, y_dev)


def test_repeated_calls_are_deterministic():
    wl = small_workload("cross4", 20, 20, 32, 16, "f32", 3, 6)
    xd = to_device(workloads.draw(wl), "f32")
    r = vs.Route("cross4", 20, 20)
    y1 = run_gpu(r, xd).clone()
    y2 = run_gpu(r, xd)
    assert torch.equal(y1, y2)


# ----------------------------------------------------------------- full-size workloads
# (workload, images sampled, channels sampled); None = all
FULL = [
    ("vim_tiny_bidir_14x14_cls", None, None),
    ("evmamba_atrous_56x56", None, None),
    ("evmamba_atrous_55x57", None, None),
    ("vmamba_ss2d_56x56_bf16", [0, 15], None),
    ("fastvim_pool_128x128", [0, 31], [0, 1, 31, 32, 100, 255, 256, 383]),
    ("vim_small_bidir_64x64_cls_bf16", [0, 63], [0, 7, 8, 300, 511, 767]),
]


@pytest.mark.parametrize("name,bsel,csel", FULL, ids=[f[0] for f in FULL])
def test_full_size_workloads(name, bsel, csel):
    wl = workloads.WORKLOADS[name]
    x = workloads.draw(wl)
    r = vs.Route(wl.route, wl.h, wl.w, wl.cls_pos)
    y = run_gpu(r, to_device(x, wl.dtype)).float().cpu().numpy()
    xs = x
    if bsel is not None:
        xs = workloads.batch_slice(xs, bsel)
        y = y[bsel]
    if csel is not None:
        xs = workloads.channel_slice(xs, csel)
        y = y[..., csel]
    ref = run_oracle(wl.route, wl.h, wl.w, wl.cls_pos, xs)
    err = rel_err(y, ref)
    assert err <= TOL[wl.dtype], (name, err)
