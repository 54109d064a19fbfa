#!/usr/bin/env python
"""Throughput of the routed visual selective scan on B200, as one JSON line.

A step is one pass of the whole fused path (gather, discretization,
recurrence, read-out, merge, gate, store) over one batch of every grid of the
selected workload. The default workload is the largest single-GPU one: the
Vim-Small-shaped high-resolution bidirectional scan (1024^2 input, 16-pixel
patches: 64x64 tokens + middle CLS = 4097 per image), batch 64, d_inner 768,
N 16, bf16 I/O with float32 state, SiLU(z) gate. Workload 1 is the
EfficientVMamba atrous p=2 scan (56x56 and the odd 55x57 grid, one step runs
both).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one process per GPU; every rank scans its own
seeded copy of the workload (weak scaling, no collective on the data path);
the timed region is bracketed by a barrier and a synchronize, and the time
is the maximum over ranks. --impl reference times the fp64 CPU oracle on the
host cores instead (rank 0 only).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "scan throughput tokens·ch/s at 1 B200; achieved HBM GB/s vs peak"
UNIT = "tokens·ch/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
TARGET_HBM_GBS = 8000.0  # the HBM roofline the >=60 % target is stated against (compulsory bytes / 8 TB/s)


def parse():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="4",
                   help="configuration index 0-4 or a workload name (default 4: Vim-Small 64x64+CLS, "
                        "b64, D768, bf16)")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU baseline budget")
    p.add_argument("--batch", type=int, default=0,
                   help="override the workload's batch (small profiling captures only)")
    p.add_argument("--rotate", type=int, default=0,
                   help="device copies of the inputs cycled through (0: enough to exceed 3x L2)")
    p.add_argument("--conv", action="store_true",
                   help="fuse the causal kernel-four Conv1d + SiLU into u (BIDIR and pooled routes)")
    p.add_argument("--zoh", action="store_true", help="zero-order-hold write term instead of Delta*B*u")
    p.add_argument("--backward", action="store_true",
                   help="time the backward pass (all gradients) instead of the forward")
    p.add_argument("--mask-keep", type=float, default=1.0,
                   help="pooled workloads: keep this fraction of tokens (random mask per image, FastMaskVim)")
    p.add_argument("--per-dir", action="store_true",
                   help="every direction its own u, raw Delta, B, C and A, D, bias planes (the Vim block's "
                        "per-branch parameters)")
    return p.parse_args()


def select(spec):
    if spec.isdigit():
        names = workloads.CONFIG_GROUPS[int(spec)]
    else:
        names = [spec]
    return [workloads.WORKLOADS[n] for n in names]


def workload_label(wls):
    w0 = wls[0]
    grids = "+".join(f"{w.h}x{w.w}" for w in wls)
    cls = "_cls" if w0.cls_pos >= 0 else ""
    opt = ("_conv" if w0.conv else "") + ("_zoh" if w0.zoh else "") + (f"_keep{w0.keep:g}" if w0.keep < 1 else "") \
        + ("_perdir" if w0.per_dir else "")
    return f"{w0.route}_{grids}{cls}_b{w0.batch}_d{w0.D}_n{w0.N}_{w0.dtype}{opt}"


def algorithmic_bytes_bwd(wl):
    """Compulsory HBM bytes of one backward: read u, raw delta, z, B, C and dy; write the
    float32 gradients du, ddelta, dz (per token-channel) and dB, dC (per token-state)."""
    eb = 2 if wl.dtype == "bf16" else 4
    ki = wl.K if wl.per_dir else 1
    per_token = (ki * (2 * wl.D + 2 * wl.N) + 2 * wl.D) * eb + (ki * (2 * wl.D + 2 * wl.N) + wl.D) * 4
    params = ki * (wl.D * wl.N + 2 * wl.D) * 4 * 2
    return wl.batch * wl.tokens * per_token + params


def algorithmic_bytes(wl):
    """Compulsory HBM bytes of one forward: read u, raw delta, B, C (one plane, or one per
    direction with per-direction inputs) and z; write y."""
    eb = 2 if wl.dtype == "bf16" else 4
    ki = wl.K if wl.per_dir else 1
    per_token = (ki * (2 * wl.D + 2 * wl.N) + wl.D) * eb + wl.D * eb
    params = ki * (wl.D * wl.N + 2 * wl.D + (5 * wl.D if wl.conv else 0)) * 4
    pos = 4 * wl.batch * wl.visible if wl.keep < 1 else 0  # grid positions of the visible tokens
    return wl.batch * wl.visible * per_token + params + pos


def seq_geometry(wl):
    K = {"bidir": 2, "cross4": 4, "atrous2": 4, "pool_w": 2, "pool_h": 2}[wl.route]
    if wl.route == "atrous2":
        L = ((wl.h + 1) // 2) * ((wl.w + 1) // 2)
    elif wl.route == "pool_w":
        L = wl.h
    elif wl.route == "pool_h":
        L = wl.w
    else:
        L = wl.tokens
    return K, L


def updates(wl):
    """Recurrence steps x states of one forward (padding steps included)."""
    K, L = seq_geometry(wl)
    return wl.batch * K * L * wl.D * wl.N


def roofline_object(bytes_all, upd_all, ms_all, hbm_peak, peak_src, sm_max, traffic, *, kernel,
                    launch_ms_avg, algorithmic_bytes, backward=False, steps=1):
    """The bench line's roofline of the dominant kernel. Both floors of the forward are
    computed, compulsory bytes at the HBM peak and one ex2 per state update at the SFU
    peak; the larger one binds. An SFU-bound forward reports "bound": "alu" against the
    SFU peak (state updates/s), with the HBM figures in the "hbm" sub-object; an HBM-bound
    one (the pooled routes) reports "hbm" with the SFU figures in "sfu". The backward pass
    is reported against HBM (its exponentials per state update depend on the recompute
    scheme, so there is no method-fixed SFU floor), with the forward-equivalent SFU rate."""
    sec = ms_all * 1e-3
    achieved = bytes_all / sec / 1e9
    upd_rate = upd_all / sec
    sfu_peak = 16 * 148 * sm_max * 1e6  # one exp per state update on the SFU
    fma_peak = 128 * 148 * sm_max * 1e6  # FP32 lane-ops/s: 128 FP32 lanes per SM
    hbm = {"achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
           "frac": round(achieved / hbm_peak, 4),
           "peak_source": f"{peak_src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
           "frac_vs_8TBs": round(achieved / TARGET_HBM_GBS, 4),
           "frac_note": "frac divides by the measured copy bandwidth; frac_vs_8TBs by the 8 TB/s "
                        "the >=60% HBM target is stated against"}
    sfu = {"state_updates_per_s": upd_rate, "peak": sfu_peak, "frac": round(upd_rate / sfu_peak, 4),
           "note": "one ex2 per state update, 16 SFU results/clk/SM x 148 SMs at max clock"}
    fp32 = {"lane_ops_per_s": 4 * upd_rate, "peak": fma_peak, "frac": round(4 * upd_rate / fma_peak, 4),
            "note": "4 FP32 ops per state update (Delta*A, Delta*u*B, the state FMA, the "
                    "read-out FMA), 128 FP32 lanes/clk/SM x 148 SMs at max clock"}
    t_hbm = bytes_all / (hbm_peak * 1e9) / steps  # per step
    t_sfu = upd_all / sfu_peak / steps
    common = {"traffic": traffic, "kernel": kernel, "launch_ms_avg": launch_ms_avg,
              "algorithmic_bytes_per_launch": algorithmic_bytes,
              "floors_ms_per_step": {"hbm": round(1e3 * t_hbm, 5), "sfu": round(1e3 * t_sfu, 5)}}
    if not backward and t_sfu > t_hbm:
        return dict({"bound": "alu", "achieved": round(upd_rate / 1e9, 1), "peak": round(sfu_peak / 1e9, 1),
                     "unit": "G state updates/s", "frac": sfu["frac"],
                     "peak_source": "SFU: 16 ex2 results/clk/SM x 148 SMs x max SM clock, one ex2 per state "
                                    "update (the method's minimum SFU work)",
                     "hbm": hbm, "fp32": fp32}, **common)
    return dict({"bound": "hbm"}, **{k: v for k, v in hbm.items()}, sfu=sfu, fp32=fp32, **common)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured", float(d.get("sm_max_mhz", 1965.0))
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback", 1965.0


# device-code files each timed kernel is compiled from (host-side API code excluded)
KERNEL_SOURCES = {
    "stream_scan_kernel": ("vscan_stream.cuh", "vscan_params.cuh", "vscan_common.cuh", "vscan_route.cuh"),
    "pipe_scan_kernel": ("vscan_pipe.cuh", "vscan_params.cuh", "vscan_common.cuh", "vscan_route.cuh"),
    "resident_scan_kernel": ("vscan_resident.cuh", "vscan_params.cuh", "vscan_common.cuh", "vscan_route.cuh"),
    "pool_scan_kernel": ("vscan_pool.cuh", "vscan_common.cuh", "vscan_route.cuh"),
    "bwd_scan_kernel": ("vscan_backward.cuh", "vscan_params.cuh", "vscan_common.cuh", "vscan_route.cuh"),
    "bwd_scan_split_kernel": ("vscan_backward.cuh", "vscan_params.cuh", "vscan_common.cuh", "vscan_route.cuh"),
}


def source_digest(kernel=None):
    """Digest of the device code a kernel is built from (all kernel headers if None)."""
    csrc = os.path.join(ROOT, "vision_selective_state_b200", "csrc")
    if kernel is None:
        names = sorted(n for n in os.listdir(csrc) if n.endswith(".cuh"))
    else:
        names = sorted(KERNEL_SOURCES[kernel.split("<")[0]])
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """dram read+write bytes per launch from a committed ncu summary, if the
    kernel sources have not changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(kernel)
    with open(path) as f:
        for ln in f:
            if ln.startswith("#") or not ln.strip():
                continue
            k, wl, dig, val = ln.split()[:4]
            if k == kernel and wl == workload and dig == digest:
                return float(val)
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML during a region."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device, interval=0.002):
        self.interval = interval
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.pci_bus_id = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle, self.pci_bus_id = self._nvml_handle(pynvml, device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.nvml = None
            self.error = str(e)

    @staticmethod
    def _nvml_handle(pynvml, device):
        """NVML handle of a torch CUDA device. CUDA and NVML number GPUs differently
        (CUDA_VISIBLE_DEVICES, fastest-first ordering), so match by UUID, else by PCI bus id."""
        import torch
        prop = torch.cuda.get_device_properties(device)
        bus = f"{prop.pci_domain_id:08x}:{prop.pci_bus_id:02x}:{prop.pci_device_id:02x}.0"
        try:
            return pynvml.nvmlDeviceGetHandleByUUID(f"GPU-{prop.uuid}"), bus
        except Exception:  # noqa: BLE001
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus), bus

    def _reason_mask(self):
        fn = getattr(self.nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(self.nvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return fn(self.handle)

    def _run(self):
        while not self._stop.is_set():
            self.sample_once()
            self._stop.wait(self.interval)

    def sample_once(self):
        if self.nvml is None:
            return
        try:
            self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
            mask = self._reason_mask()
            for bit, name in self.REASONS.items():
                if mask & bit:
                    self.reasons.add(name)
        except Exception:  # noqa: BLE001
            pass

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        self.sample_once()

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": getattr(self, "error", "nvml unavailable")}
        reasons = sorted(self.reasons - {"gpu_idle"})
        return {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "pci_bus_id": self.pci_bus_id,
                "source": f"nvml (device matched by UUID / PCI bus id), {1e3 * self.interval:g} ms "
                          f"interval, during the timed region"}


# ------------------------------------------------------------------ distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def replica(wl, rank):
    """The workload one rank scans: same shapes, its own seeded values."""
    return wl.with_(seed=wl.seed + 1000 * rank)


def max_over_ranks(value, device=None):
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, steps, world, elapsed_ms_max):
    """Whole-job throughput: units every rank processed / the slowest rank's time."""
    return units_per_rank_step * steps * world / (elapsed_ms_max * 1e-3)


# ------------------------------------------------------------------ inputs
_DRAWN = {}


def draw_inputs(wl):
    """The seeded inputs of one workload (numpy, float32), drawn once per process."""
    key = (wl.name, wl.seed, wl.batch, wl.keep, wl.conv, wl.per_dir)
    if key not in _DRAWN:
        if wl.keep < 1:
            x = workloads.draw_masked(wl)
        else:
            x = workloads.draw(wl, per_dir_inputs=wl.per_dir, per_dir_params=wl.per_dir)
        if wl.conv:
            x.update(workloads.draw_conv(wl, per_dir_params=wl.per_dir))
        _DRAWN[key] = x
    return _DRAWN[key]


# ------------------------------------------------------------------ CPU oracle
def oracle_inputs(wls, channels):
    """Every grid's inputs restricted to a channel subset (channels are independent)."""
    return [workloads.channel_slice(draw_inputs(wl), channels) for wl in wls]


def oracle_time(wls, xs, threads=0):
    """Seconds the fp64 oracle takes for the given (channel-sliced) inputs of every grid."""
    import oracle
    total = 0.0
    for wl, x in zip(wls, xs):
        t0 = time.perf_counter()
        if wl.keep < 1:
            oracle.forward_masked(wl.route, wl.h, wl.w, x["pos"], x["u"], x["delta"], x["A"], x["B"], x["C"],
                                  x["Dskip"], x["bias"], x["z"] if wl.gate else None, zoh=wl.zoh,
                                  threads=threads)
        else:
            oracle.forward(wl.route, wl.h, wl.w, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"],
                           x["bias"], x["z"] if wl.gate else None, cls_pos=wl.cls_pos,
                           conv_w=x.get("conv_w"), conv_b=x.get("conv_b"), zoh=wl.zoh,
                           per_dir_inputs=wl.per_dir, per_dir_params=wl.per_dir, threads=threads)
        total += time.perf_counter() - t0
    return total


def cpu_baseline(wls, budget_s):
    """The oracle as it stands, on the host cores, on a bounded channel sample."""
    import oracle
    cores = oracle.default_threads()
    D = wls[0].D
    n1 = min(cores, D)
    t1 = oracle_time(wls, oracle_inputs(wls, list(range(n1))))
    per_channel = t1 / n1
    nch = int(max(1, min(D, budget_s / max(per_channel, 1e-9))))
    xs = oracle_inputs(wls, list(range(nch)))
    # repeat whole passes over the sample until the budget is spent (at least one)
    t, passes = 0.0, 0
    while passes == 0 or t < budget_s:
        t += oracle_time(wls, xs)
        passes += 1
    units = sum(w.batch * w.visible * nch for w in wls) * passes
    return {"value": units / t, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"all images and tokens of every grid, {nch} of {D} channels, "
                      f"{passes} pass(es), fp64",
            "seconds": round(t, 3)}


def run_reference(args, wls):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    cores = oracle.default_threads()
    D = wls[0].D
    probe = oracle_time(wls, oracle_inputs(wls, [0]))
    steps_total = args.steps + args.warmup
    budget = 150.0  # seconds for the whole run
    nch = int(max(1, min(D, budget / steps_total / max(probe, 1e-6))))
    xs = oracle_inputs(wls, list(range(nch)))
    for _ in range(args.warmup):
        oracle_time(wls, xs)
    t = 0.0
    for _ in range(args.steps):
        t += oracle_time(wls, xs)
    units = sum(w.batch * w.visible * nch for w in wls) * args.steps
    value = units / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic, seeded (page-workload shapes and value recipe)",
        "config": config_block(wls, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: all images and tokens of every grid, {nch} of {D} channels"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(wls, n):
    w0 = wls[0]
    return {"workload": workload_label(wls), "route": w0.route,
            "grids": [f"{w.h}x{w.w}" for w in wls], "batch": w0.batch, "d_inner": w0.D,
            "d_state": w0.N, "io_dtype": w0.dtype, "gate": w0.gate, "merge_scale": w0.merge_scale,
            "conv": w0.conv, "zoh": w0.zoh, "mask_keep": w0.keep, "per_direction_planes": w0.per_dir,
            "pass": "forward",
            "parallelism": f"replicas x{n} (one full workload per GPU, no collective)"}


# ------------------------------------------------------------------ our path
def run_ours(args, wls):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:  # one process per GPU; the device is bound before the communicator
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    import vision_selective_state_b200 as vs

    stream = torch.cuda.Stream(dev)
    td = {"f32": torch.float32, "bf16": torch.bfloat16}
    # Rotate several device copies of every input so that no step finds its
    # inputs in the 126 MB L2 left by the previous step.
    step_bytes = sum(algorithmic_bytes(w) for w in wls)
    rot = max(2, -(-3 * L2_BYTES // step_bytes) + 1)
    rot = min(rot, 8) if args.rotate <= 0 else args.rotate
    plans, host_sets, routes = [], [], []
    for wi, wl in enumerate(wls):
        x = draw_inputs(replica(wl, rank))
        route = vs.Route(wl.route, wl.h, wl.w, wl.cls_pos)
        routes.append(route)
        dt = td[wl.dtype]
        host = {k: torch.from_numpy(x[k]).to(dt) for k in ("u", "delta", "B", "C", "z")}
        host.update({k: torch.from_numpy(np.ascontiguousarray(x[k], dtype=np.float32))
                     for k in ("A", "Dskip", "bias") + (("conv_w", "conv_b") if wl.conv else ())})
        if wl.keep < 1:
            host["pos"] = torch.from_numpy(x["pos"])
        host_sets.append(host)
        pd = dict(per_dir_inputs=wl.per_dir, per_dir_params=wl.per_dir)
        ws_bytes = vs.workspace_size(route, host["u"], host["B"], token_pos=host.get("pos"), **pd)
        per = []
        for r in range(rot):
            d = {k: v.to(dev) for k, v in host.items()}
            ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
            if args.backward:
                dy = torch.randn(d["u"].shape[-3:], generator=torch.Generator().manual_seed(rank)).to(
                    dev, d["u"].dtype)
                per.append(vs.BackwardPlan(route, d["u"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"],
                                           d["bias"], d["z"] if wl.gate else None, dy=dy,
                                           merge_scale=wl.merge_scale, **pd))
                continue
            out = torch.empty(d["z"].shape, dtype=d["u"].dtype, device=dev)
            per.append(vs.Plan(route, d["u"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], d["bias"],
                               d["z"] if wl.gate else None, out=out, workspace=ws,
                               merge_scale=wl.merge_scale, conv_w=d.get("conv_w"),
                               conv_b=d.get("conv_b"), zoh=wl.zoh, token_pos=d.get("pos"), **pd))
        plans.append(per)
    launches_per_step = sum(per[0].kernels() for per in plans)
    knames = sorted({per[0].kernel_name() for per in plans})
    torch.cuda.synchronize(dev)

    # warm-up
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            for per in plans:
                per[i % rot].run(stream)
    stream.synchronize()

    K = args.steps
    nfw = len(wls)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(nfw)] for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    wall0 = time.perf_counter()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(K):
            for j, per in enumerate(plans):
                a, b = ev[i][j]
                a.record(stream)
                per[i % rot].run(stream)
                b.record(stream)
        t_end.record(stream)
    stream.synchronize()
    wall = time.perf_counter() - wall0
    sampler.stop()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    per_launch_ms = [[ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(K)] for j in range(nfw)]
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)

    units_step = sum(w.token_channels for w in wls)
    value = job_throughput(units_step, K, world, elapsed_ms)

    # roofline of the dominant kernel (the fused scan: one launch per forward for
    # the streaming routes; for the pooled route the bracket also holds the small
    # B/C pooling pre-pass)
    hbm_peak, peak_src, sm_max = peaks()
    ab = algorithmic_bytes_bwd if args.backward else algorithmic_bytes
    bytes_all = sum(ab(w) * K for w in wls)
    ms_all = sum(sum(v) for v in per_launch_ms)
    kname = "+".join(knames)
    traffic = recorded_traffic(kname, workload_label(wls))
    upd_all = sum(updates(w) * K for w in wls)
    roofline = roofline_object(bytes_all, upd_all, ms_all, hbm_peak, peak_src, sm_max, traffic,
                               kernel=kname, launch_ms_avg=round(ms_all / (K * nfw), 5),
                               algorithmic_bytes=[ab(w) for w in wls], backward=args.backward, steps=K)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if wls[0].dtype == "f32" else "bf16",
        "data": "synthetic, seeded (page-workload shapes and value recipe)",
        "config": dict(config_block(wls, world), **({"pass": "backward (all gradients)"} if args.backward else {}),
                       l2=f"rotating {rot} device copies of the inputs ({rot * step_bytes / 2**20:.0f} MiB; "
                          f"each step's inputs were last touched {rot - 1} steps earlier)"),
        "roofline": roofline,
        "gpu_launches": K * launches_per_step,
        "clocks": sampler.summary(),
        "wall_s_timed_region": round(wall, 4),
    }

    # end to end through the host-buffer entry point: two streams, each with its
    # own device buffer and host output, so the copies of one step overlap the
    # scan and the copy-back of the other (a user's pipelined loop)
    if not args.no_e2e:
        streams = [stream, torch.cuda.Stream(dev)]
        hplans, h2d, d2h = [[], []], 0, 0
        for wl, route, host in zip(wls, routes, host_sets):
            pin = {k: v.pin_memory() for k, v in host.items()}
            pd = dict(per_dir_inputs=wl.per_dir, per_dir_params=wl.per_dir)
            nbytes = vs.host_buffer_size(route, pin["u"], pin["B"], z=wl.gate, conv_w=wl.conv,
                                         conv_b=wl.conv, token_pos=wl.keep < 1, **pd)
            for slot in range(2):
                out = torch.empty(pin["z"].shape, dtype=pin["u"].dtype).pin_memory()
                buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
                hplans[slot].append(vs.HostPlan(route, pin["u"], pin["delta"], pin["A"], pin["B"], pin["C"],
                                                pin["Dskip"], pin["bias"], pin["z"] if wl.gate else None,
                                                out=out, device_buffer=buf, merge_scale=wl.merge_scale,
                                                conv_w=pin.get("conv_w"), conv_b=pin.get("conv_b"),
                                                zoh=wl.zoh, token_pos=pin.get("pos"), **pd))
            h2d += sum(v.numel() * v.element_size() for k, v in pin.items() if k != "z" or wl.gate)
            d2h += hplans[0][-1].out.numel() * hplans[0][-1].out.element_size()
        E = max(2, min(args.e2e_steps, K))
        for slot in range(2):  # warm-up of both slots
            for hp in hplans[slot]:
                hp.run(streams[slot])
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        done_b = torch.cuda.Event()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0.record(streams[0])
        streams[1].wait_event(e0)
        for i in range(E):
            for hp in hplans[i % 2]:
                hp.run(streams[i % 2])
        done_b.record(streams[1])
        streams[0].wait_event(done_b)
        e1.record(streams[0])
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        line["e2e"] = {"value": job_throughput(units_step, E, world, e_ms), "unit": UNIT,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": E,
                       "path": "vscan_forward_host (pinned host buffers, copies inside the timed region; "
                               "two streams alternate steps so copies overlap the scan)"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wls, args.cpu_seconds)

    if rank == 0:
        print(json.dumps(line), flush=True)
    for r in routes:
        r.close()
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    wls = select(args.workload)
    if args.batch > 0:
        wls = [w.with_(batch=args.batch) for w in wls]
    if args.backward and (args.conv or args.zoh or args.mask_keep < 1):
        raise SystemExit("--backward covers the Delta*B*u scan without --conv, --zoh or --mask-keep")
    if args.per_dir:
        if args.mask_keep < 1:
            raise SystemExit("--per-dir does not combine with --mask-keep")
        wls = [w.with_(per_dir=True) for w in wls]
    if args.backward:
        args.no_e2e = True  # the end-to-end leg times the forward entry point
    if args.conv or args.zoh or args.mask_keep < 1:
        wls = [w.with_(conv=args.conv, zoh=args.zoh, keep=args.mask_keep) for w in wls]
        if args.mask_keep < 1 and (wls[0].route not in ("pool_w", "pool_h") or args.conv):
            raise SystemExit("--mask-keep applies to the pooled workload (3), without --conv")
        if args.conv and wls[0].route in ("cross4", "atrous2"):
            raise SystemExit("--conv applies to the bidir and pooled workloads (0, 3, 4)")
    if args.impl == "reference":
        run_reference(args, wls)
    else:
        run_ours(args, wls)


if __name__ == "__main__":
    main()
