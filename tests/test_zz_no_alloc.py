"""vscan_forward_pooled_noalloc: the pooled-route forward pass that allocates nothing.

Some callers cannot allocate device memory: a plugin whose host runtime owns all
device memory, or a latency-bound loop that must not call cudaMalloc (it can
synchronize the device and fail under memory pressure). For them the library
keeps the pooled route's only scratch (the pooled B and C) in a fixed 4 MiB
device array. This test calls that entry point through the C ABI and checks its
output against vscan_forward's on the same inputs, on two calls in a row with
different inputs (the shared array keeps the previous call's contents, which
must not leak into the next result). It runs last, alone or after the others.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import workloads
from vscan_testlib import TOL, rel_err, to_device

import vision_selective_state_b200 as vs
from vision_selective_state_b200 import _abi

pytestmark = pytest.mark.gpu


def _noalloc(route, xd, out):
    a = vs._args(route, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
                 out, True, 1.0, False, False, None, 0)
    stream = torch.cuda.current_stream()
    _abi.check(_abi.lib.vscan_forward_pooled_noalloc(route.handle, ctypes.byref(a),
                                                     ctypes.c_void_p(stream.cuda_stream)))
    return out


@pytest.mark.parametrize("route,h,w,batch,D,dtype", [
    ("pool_w", 128, 128, 4, 64, "f32"),
    ("pool_h", 24, 40, 3, 48, "bf16"),
])
def test_noalloc_matches_forward_on_two_calls(route, h, w, batch, D, dtype):
    r = vs.Route(route, h, w)
    for call, seed in enumerate((101, 202)):
        wl = workloads.Workload(f"noalloc_{call}", route, h, w, -1, batch, D, 16, dtype, seed)
        xd = to_device(workloads.draw(wl, a_mode="random"), dtype)
        ref = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"])
        got = _noalloc(r, xd, torch.empty_like(ref))
        torch.cuda.synchronize()
        err = rel_err(got.float().cpu().numpy(), ref.float().cpu().numpy())
        assert err <= TOL[dtype], (route, call, err)
    r.close()
