"""vscan_forward_pooled_noalloc: the pooled-route forward pass that allocates nothing.

Some callers cannot allocate device memory: a plugin whose host runtime owns all
device memory, or a latency-bound loop that must not call cudaMalloc (it can
synchronize the device and fail under memory pressure). For them the library
keeps the pooled route's only scratch (the pooled B and C) in a fixed 4 MiB
device array. This test calls that entry point through the C ABI and checks its
output against vscan_forward's and against the fp64 oracle on the same inputs,
on two calls in a row with different inputs (the shared array keeps the previous
call's contents, which must not leak into the next result). The masked case
accumulates its pooled sums in the array, so it also checks that the call clears
what it uses. It runs last, alone or after the others.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import oracle as O
import workloads
from vscan_testlib import TOL, rel_err, to_device

import vision_selective_state_b200 as vs
from vision_selective_state_b200 import _abi

pytestmark = pytest.mark.gpu


def _noalloc(route, xd, out, token_pos=None):
    a = vs._args(route, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
                 out, True, 1.0, False, False, None, 0, None, None, False, token_pos)
    stream = torch.cuda.current_stream()
    _abi.check(_abi.lib.vscan_forward_pooled_noalloc(route.handle, ctypes.byref(a),
                                                     ctypes.c_void_p(stream.cuda_stream)))
    return out


@pytest.mark.parametrize("route,h,w,batch,D,dtype,keep", [
    ("pool_w", 128, 128, 4, 64, "f32", 1.0),
    ("pool_h", 24, 40, 3, 48, "bf16", 1.0),
    ("pool_w", 32, 48, 3, 32, "f32", 0.3),
])
def test_noalloc_matches_forward_and_oracle_on_two_calls(route, h, w, batch, D, dtype, keep):
    r = vs.Route(route, h, w)
    for call, seed in enumerate((101, 202)):
        wl = workloads.Workload(f"noalloc_{call}", route, h, w, -1, batch, D, 16, dtype, seed)
        pos = tp = None
        if keep < 1:
            n = max(1, int(round(keep * h * w)))
            x = workloads.draw(wl.with_(h=n, w=1), a_mode="random")
            rng = np.random.default_rng(seed + 1)
            pos = np.stack([np.sort(rng.choice(h * w, n, replace=False)) for _ in range(batch)]).astype(np.int32)
            tp = torch.from_numpy(pos).cuda()
        else:
            x = workloads.draw(wl, a_mode="random")
        xd = to_device(x, dtype)
        ref = vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
                         token_pos=tp)
        got = _noalloc(r, xd, torch.empty_like(ref), tp)
        torch.cuda.synchronize()
        g = got.float().cpu().numpy()
        err = rel_err(g, ref.float().cpu().numpy())
        assert err <= TOL[dtype], (route, call, "vs vscan_forward", err)
        if keep < 1:
            yo = O.forward_masked(route, h, w, pos, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"],
                                  x["bias"], x["z"])
        else:
            yo = O.forward(route, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"], x["z"])
        err_o = rel_err(g, yo)
        assert err_o <= TOL[dtype], (route, call, "vs oracle", err_o)
    r.close()
