"""The mbarrier-pipelined kernel (BIDIR and CROSS4 with d_state 16) against the
fp64 oracle, and the device status word.

seq_chunks=1 keeps every case on the streaming path, which for these routes is
pipe_scan_kernel: ragged last chunks (sequence lengths 1 .. 1601, not multiples
of the 16-step chunk), partial channel tiles (D not a multiple of the 8- or
16-channel tile), tokens whose directions meet in the same chunk and in chunks
far apart (the two merge sources), both I/O types, shared and per-direction
inputs and parameters, and every optional term.

The status word: zero after a clean call; VSCAN_FLAG_CHECK_VALUES flags a NaN
input, an unstable A (> 0), a negative time scale with softplus off, and leaves
finite inputs alone.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import workloads
from vscan_testlib import TOL, rel_err, run_gpu, run_oracle, small_workload, to_device

import vision_selective_state_b200 as vs

pytestmark = pytest.mark.gpu


def _case(route, h, w, D, dtype, batch=2, seed=3, pdi=False, pdp=False, cls=None, **opts):
    wl = small_workload(route, h, w, D, 16, dtype, batch, seed, cls)
    x = workloads.draw(wl, a_mode="random", per_dir_inputs=pdi, per_dir_params=pdp)
    if opts.get("delta_softplus") is False:
        x["delta"] = np.abs(x["delta"])
        x["bias"] = np.full_like(x["bias"], 0.01)
    r = vs.Route(route, h, w, wl.cls_pos)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = run_gpu(r, to_device(x, dtype), per_dir_inputs=pdi, per_dir_params=pdp, seq_chunks=1, status=status,
                **opts)
    assert int(status.item()) == 0
    ref = run_oracle(route, h, w, wl.cls_pos, x, per_dir_inputs=pdi, per_dir_params=pdp, **opts)
    err = rel_err(y.float().cpu().numpy(), ref)
    assert err <= TOL[dtype], (route, h, w, D, dtype, err)


def test_pipelined_kernel_is_the_streaming_choice():
    for kind, h, w in (("bidir", 9, 13), ("cross4", 9, 13)):
        r = vs.Route(kind, h, w, (h * w) // 2 if kind == "bidir" else -1)
        wl = small_workload(kind, h, w, 16, 16, "bf16", 2, 1)
        xd = to_device(workloads.draw(wl), "bf16")
        out = torch.empty_like(xd["u"])
        ws = torch.empty(max(1, vs.workspace_size(r, xd["u"], xd["B"])), dtype=torch.uint8, device="cuda")
        plan = vs.Plan(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
                       out=out, workspace=ws, seq_chunks=1)
        assert plan.kernel_name() == f"pipe_scan_kernel<{kind.upper()}>"


@pytest.mark.parametrize("route", ["bidir", "cross4"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("h,w", [(1, 1), (1, 9), (9, 1), (3, 5), (6, 4), (13, 11), (16, 17), (5, 33)])
def test_ragged_chunks(route, dtype, h, w):
    _case(route, h, w, 16, dtype)


@pytest.mark.parametrize("route", ["bidir", "cross4"])
@pytest.mark.parametrize("D,dtype", [(8, "bf16"), (24, "bf16"), (40, "bf16"), (4, "f32"), (12, "f32"), (36, "f32")])
def test_partial_channel_tiles(route, D, dtype):
    _case(route, 7, 10, D, dtype)


@pytest.mark.parametrize("route", ["bidir", "cross4"])
def test_per_direction_planes(route):
    _case(route, 9, 7, 16, "f32", pdi=True, pdp=True)
    _case(route, 9, 7, 24, "bf16", pdi=False, pdp=True)
    _case(route, 9, 7, 16, "bf16", pdi=True, pdp=False)


@pytest.mark.parametrize("route", ["bidir", "cross4"])
def test_optional_terms(route):
    _case(route, 8, 9, 16, "f32", gate=False)
    _case(route, 8, 9, 16, "f32", skip=False, bias=False)
    _case(route, 8, 9, 16, "bf16", merge_scale=0.5)
    _case(route, 8, 9, 16, "f32", delta_softplus=False)


def test_long_sequences():
    _case("bidir", 40, 40, 24, "f32", batch=1)             # L = 1601, CLS 800
    _case("bidir", 45, 46, 16, "bf16", batch=1, cls=1035)   # L = 2071
    _case("bidir", 32, 64, 32, "bf16", batch=1, cls=-1)     # L = 2048, an exact multiple
    _case("cross4", 31, 33, 8, "bf16", batch=1)             # L = 1023
    _case("cross4", 40, 24, 16, "f32", batch=2)             # column-major chunks across columns


def _value_case(mutate, softplus=True):
    wl = small_workload("cross4", 6, 7, 16, 16, "f32", 2, 9)
    x = workloads.draw(wl)
    mutate(x)
    xd = to_device(x, "f32")
    r = vs.Route("cross4", 6, 7)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
               delta_softplus=softplus, status=status, check_values=True)
    torch.cuda.synchronize()
    return int(status.item())


def test_value_checks_flag_bad_inputs_and_pass_clean_ones():
    """EfficientVMamba review, sec. 2: the scalar scan refuses non-finite inputs, an unstable A and
    negative time scales. Here they set bit 1 of the status word instead, and clean inputs leave it 0."""
    assert _value_case(lambda x: None) == 0
    assert _value_case(lambda x: x["u"].__setitem__((1, 5, 3), np.nan)) == 1
    assert _value_case(lambda x: x["B"].__setitem__((0, 0, 15), np.inf)) == 1
    assert _value_case(lambda x: x["z"].__setitem__((0, 41, 0), -np.inf)) == 1
    assert _value_case(lambda x: x["A"].__setitem__((2, 7), 0.25)) == 1
    assert _value_case(lambda x: x["bias"].__setitem__(4, np.nan)) == 1
    # softplus off: Delta = raw + bias must be >= 0
    def positive(x):
        x["delta"][:] = np.abs(x["delta"])
        x["bias"][:] = 0.0
    assert _value_case(positive, softplus=False) == 0

    def negative(x):
        positive(x)
        x["delta"][1, 40, 9] = -1e-3
    assert _value_case(negative, softplus=False) == 1
    assert vs.status_from_device_word(0) == 0
    assert vs.status_from_device_word(1) == -7   # VSCAN_ERR_VALUE
    assert vs.status_from_device_word(2) == -8   # VSCAN_ERR_DEVICE_TIMEOUT
    assert vs.status_from_device_word(3) == -8


def test_value_checks_need_a_status_word():
    wl = small_workload("bidir", 3, 3, 8, 16, "f32", 1, 2)
    xd = to_device(workloads.draw(wl), "f32")
    r = vs.Route("bidir", 3, 3, 4)
    with pytest.raises(vs.VscanError):
        vs.forward(r, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], xd["Dskip"], xd["bias"], xd["z"],
                   check_values=True)
