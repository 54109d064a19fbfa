"""vscan_forward inside a captured CUDA graph.

A forward call enqueues only kernel launches on the caller's stream (no
allocation, no synchronization), so it can be captured once and replayed: after
new values are copied into the captured input buffers, a replay must give the
same output as an eager call on those values, bit for bit. Covers the
pipelined (BIDIR, CROSS4), streaming (ATROUS2), resident (small BIDIR) and
pooled kernels, and a strided call (pack kernels in the graph).
"""
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import workloads
from vscan_testlib import small_workload, to_device

import vision_selective_state_b200 as vs

pytestmark = pytest.mark.gpu


def _inputs(route, h, w, D, dtype, batch, seed):
    wl = small_workload(route, h, w, D, 16, dtype, batch, seed)
    return wl, to_device(workloads.draw(wl, a_mode="random"), dtype)


@pytest.mark.parametrize("route,h,w,D,dtype,batch,chunks", [
    ("bidir", 16, 16, 32, "bf16", 4, 1),     # pipelined
    ("cross4", 12, 10, 16, "bf16", 3, 1),    # pipelined
    ("atrous2", 9, 11, 24, "f32", 2, 1),     # streaming
    ("bidir", 7, 7, 64, "f32", 1, 4),        # resident chunked scan
    ("pool_w", 16, 12, 32, "f32", 2, 0),     # pooled
])
def test_replayed_graph_matches_eager_calls(route, h, w, D, dtype, batch, chunks):
    wl, x = _inputs(route, h, w, D, dtype, batch, seed=3)
    r = vs.Route(route, h, w, wl.cls_pos)
    out = torch.empty_like(x["z"])
    ws = torch.empty(max(16, vs.workspace_size(r, x["u"], x["B"])), dtype=torch.uint8, device="cuda")

    def call():
        vs.forward(r, x["u"], x["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"], x["z"], out=out,
                   workspace=ws, seq_chunks=chunks)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()  # first call outside the capture (one-time attribute setup)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for seed in (5, 7):
        _, x2 = _inputs(route, h, w, D, dtype, batch, seed)
        for k in ("u", "delta", "B", "C", "z", "A", "Dskip", "bias"):
            x[k].copy_(x2[k])
        g.replay()
        torch.cuda.synchronize()
        eager = vs.forward(r, x2["u"], x2["delta"], x2["A"], x2["B"], x2["C"], x2["Dskip"], x2["bias"], x2["z"],
                           seq_chunks=chunks)
        torch.cuda.synchronize()
        assert torch.equal(out, eager), (route, seed)


def test_replayed_graph_with_strided_views():
    route, h, w, D, dtype, batch = "bidir", 8, 8, 16, "f32", 2
    wl, x = _inputs(route, h, w, D, dtype, batch, seed=3)
    r = vs.Route(route, h, w, wl.cls_pos)
    big = {k: torch.zeros(batch, x[k].shape[1] + 1, x[k].shape[2] + 8, device="cuda") for k in ("u", "delta", "z")}
    v = {k: big[k][:, : x[k].shape[1], : x[k].shape[2]] for k in big}
    ybig = torch.zeros_like(big["z"])
    y = ybig[:, : x["z"].shape[1], : x["z"].shape[2]]
    ws = torch.empty(vs.workspace_size(r, v["u"], x["B"], z=v["z"]), dtype=torch.uint8, device="cuda")

    def call():
        vs.forward(r, v["u"], v["delta"], x["A"], x["B"], x["C"], x["Dskip"], x["bias"], v["z"], out=y, workspace=ws)

    for k in v:
        v[k].copy_(x[k])
    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    _, x2 = _inputs(route, h, w, D, dtype, batch, seed=9)
    for k in v:
        v[k].copy_(x2[k])
    for k in ("B", "C", "A", "Dskip", "bias"):
        x[k].copy_(x2[k])
    g.replay()
    torch.cuda.synchronize()
    eager = vs.forward(r, x2["u"], x2["delta"], x2["A"], x2["B"], x2["C"], x2["Dskip"], x2["bias"], x2["z"])
    torch.cuda.synchronize()
    assert torch.equal(y, eager)
