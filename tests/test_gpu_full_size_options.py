"""The optional steps and the backward pass at the full workload sizes, in the
launch configuration bench.py times, checked on sampled images and channels
(images are independent, and so are channels except for the dB / dC gradients,
which are compared on whole images).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import oracle as O
import workloads
from vscan_testlib import TOL, rel_err, to_device

import vision_selective_state_b200 as vs

pytestmark = pytest.mark.gpu


def _slices(x, bsel, csel):
    xs = workloads.batch_slice(x, bsel) if bsel is not None else dict(x)
    if "pos" in x and bsel is not None:
        xs["pos"] = np.ascontiguousarray(x["pos"][bsel])
    if csel is not None:
        xs = workloads.channel_slice(xs, csel)
    return xs


# (workload, option, images sampled, channels sampled)
FWD = [
    ("vim_small_bidir_64x64_cls_bf16", "conv", [0, 63], [0, 7, 8, 300, 511, 767]),
    ("fastvim_pool_128x128", "conv", [0, 31], [0, 1, 31, 32, 200, 383]),
    ("evmamba_atrous_56x56", "zoh", None, None),
    ("vmamba_ss2d_56x56_bf16", "zoh", [0, 15], None),
    ("fastvim_pool_128x128", "mask", [0, 31], [0, 1, 31, 32, 200, 383]),
]


@pytest.mark.parametrize("name,opt,bsel,csel", FWD, ids=[f"{f[0]}-{f[1]}" for f in FWD])
def test_full_size_options(name, opt, bsel, csel):
    wl = workloads.WORKLOADS[name]
    if opt == "mask":
        wl = wl.with_(keep=0.25)
        x = workloads.draw_masked(wl)
    else:
        x = workloads.draw(wl)
    if opt == "conv":
        x.update(workloads.draw_conv(wl))
    xd = to_device(x, wl.dtype)
    r = vs.Route(wl.route, wl.h, wl.w, wl.cls_pos)
    kw = {}
    if opt == "conv":
        kw = dict(conv_w=torch.from_numpy(x["conv_w"]).cuda(), conv_b=torch.from_numpy(x["conv_b"]).cuda())
    elif opt == "zoh":
        kw = dict(zoh=True)
    elif opt == "mask":
        kw = dict(token_pos=torch.from_numpy(x["pos"]).cuda())
    y = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"], **kw)
    torch.cuda.synchronize()
    y = y.float().cpu().numpy()
    if bsel is not None:
        y = y[bsel]
    if csel is not None:
        y = y[..., csel]
    xs = _slices(x, bsel, csel)
    if opt == "mask":
        ref = O.forward_masked(wl.route, wl.h, wl.w, xs["pos"], xs["u"], xs["delta"], xs["A"], xs["B"], xs["C"],
                               xs["Dskip"], xs["bias"], xs["z"])
    else:
        ref = O.forward(wl.route, wl.h, wl.w, xs["u"], xs["delta"], xs["A"], xs["B"], xs["C"], xs["Dskip"],
                        xs["bias"], xs["z"], cls_pos=wl.cls_pos, conv_w=xs.get("conv_w"),
                        conv_b=xs.get("conv_b"), zoh=opt == "zoh")
    err = rel_err(y, ref)
    assert err <= TOL[wl.dtype], (name, opt, err)


# backward: (workload, images sampled)
BWD = [("evmamba_atrous_56x56", None), ("vmamba_ss2d_56x56_bf16", [0, 15]),
       ("fastvim_pool_128x128", [0, 31]), ("vim_small_bidir_64x64_cls_bf16", [0, 63])]


@pytest.mark.parametrize("name,bsel", BWD, ids=[b[0] for b in BWD])
def test_full_size_backward(name, bsel):
    wl = workloads.WORKLOADS[name]
    x = workloads.draw(wl)
    dy = np.random.default_rng(wl.seed + 5).standard_normal((wl.batch, wl.tokens, wl.D)).astype(np.float32)
    if wl.dtype == "bf16":
        dy = workloads.round_to_bf16(dy)
    xd = to_device(x, wl.dtype)
    r = vs.Route(wl.route, wl.h, wl.w, wl.cls_pos)
    g = vs.backward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
                    dy=torch.from_numpy(dy).to("cuda", xd["u"].dtype))
    torch.cuda.synchronize()
    xs = _slices(x, bsel, None)
    dys = dy if bsel is None else np.ascontiguousarray(dy[bsel])
    ref = O.backward(wl.route, wl.h, wl.w, xs["u"], xs["delta"], xs["A"], xs["B"], xs["C"], xs["Dskip"],
                     xs["bias"], xs["z"], dy=dys, cls_pos=wl.cls_pos)
    for k in ("du", "ddelta", "dB", "dC", "dz"):
        got = g[k].cpu().numpy()
        if bsel is not None:
            got = got[bsel]
        assert rel_err(got, ref[k]) <= TOL[wl.dtype], (name, k)
    if bsel is None:  # parameter gradients sum over every image
        for k in ("dA", "dDskip", "dbias"):
            assert rel_err(g[k].cpu().numpy(), ref[k]) <= TOL[wl.dtype], (name, k)
