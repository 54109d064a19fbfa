"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the binding, run the oracle on the same values and
compare with the tolerance metric.

Tolerance metric: err = max_i |y_i - yref_i| / max(|yref_i|, rms(yref)), i.e. a
relative error that falls back to the output's RMS where the reference crosses
zero (the gated output is signed). Bounds: 1e-4 for float32 I/O, 2e-2 for
bfloat16 I/O with float32 state.
"""
import numpy as np
import torch

import oracle as O
import workloads

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    denom = np.maximum(np.abs(ref), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(y - ref) / denom))


def torch_dtype(dt):
    return torch.bfloat16 if dt == "bf16" else torch.float32


def to_device(x, dtype, device="cuda"):
    td = torch_dtype(dtype)
    out = {}
    for k in ("u", "delta", "B", "C", "z"):
        if x.get(k) is not None:
            out[k] = torch.from_numpy(np.ascontiguousarray(x[k])).to(device=device, dtype=td)
    for k in ("A", "Dskip", "bias"):
        if x.get(k) is not None:
            out[k] = torch.from_numpy(np.ascontiguousarray(x[k], dtype=np.float32)).to(device)
    return out


def run_gpu(route, xd, *, gate=True, skip=True, bias=True, **kw):
    import vision_selective_state_b200 as vs
    y = vs.forward(route, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                   xd["Dskip"] if skip else None, xd["bias"] if bias else None,
                   xd["z"] if gate else None, **kw)
    torch.cuda.synchronize()
    return y


def run_oracle(kind, h, w, cls, x, *, gate=True, skip=True, bias=True, delta_softplus=True,
               merge_scale=1.0, per_dir_inputs=False, per_dir_params=False):
    return O.forward(kind, h, w, x["u"], x["delta"], x["A"], x["B"], x["C"],
                     x["Dskip"] if skip else None, x["bias"] if bias else None,
                     x["z"] if gate else None, cls_pos=cls, delta_softplus=delta_softplus,
                     merge_scale=merge_scale, per_dir_inputs=per_dir_inputs,
                     per_dir_params=per_dir_params)


def small_workload(route, h, w, D, N, dtype, batch, seed, cls=None):
    if cls is None:
        cls = (h * w) // 2 if route == "bidir" else -1
    return workloads.Workload(f"{route}_{h}x{w}", route, h, w, cls, batch, D, N, dtype, seed)
