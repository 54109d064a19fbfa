"""The bench line's roofline object (host only): which bound binds each workload and the
fields it carries.

For the five page workloads the method's own floors are fixed by their sizes: compulsory
bytes at the HBM peak, and one ex2 per state update at the SFU peak (16 results per clock
and SM, 148 SMs). The pooled FastVim route scans 1/128 of its tokens, so HBM binds; every
other route issues one SFU op per state for 8-16 bytes of traffic per 16 states, so the SFU
binds and the line reports "alu" against the SFU peak, keeping the HBM fraction beside it.
"""
import bench
import workloads

SM_MAX = 1965.0
HBM = 6650.0


def _roof(idx, ms=1.0, backward=False, steps=1):
    """Roofline of `steps` timed steps of config idx taking ms each."""
    wls = [workloads.WORKLOADS[n] for n in workloads.CONFIG_GROUPS[idx]]
    ab = bench.algorithmic_bytes_bwd if backward else bench.algorithmic_bytes
    bytes_all = sum(ab(w) for w in wls) * steps
    upd_all = sum(bench.updates(w) for w in wls) * steps
    return bench.roofline_object(bytes_all, upd_all, ms * steps, HBM, "fallback", SM_MAX, None, kernel="k",
                                 launch_ms_avg=ms, algorithmic_bytes=[ab(w) for w in wls], backward=backward,
                                 steps=steps)


def test_sfu_bound_workloads_report_alu_against_the_sfu_peak():
    for idx in (0, 1, 2, 4):
        r = _roof(idx)
        assert r["bound"] == "alu", idx
        assert r["floors_ms_per_step"]["sfu"] > r["floors_ms_per_step"]["hbm"], idx
        sfu_peak_g = 16 * 148 * SM_MAX * 1e6 / 1e9
        assert r["peak"] == round(sfu_peak_g, 1)
        # achieved = state updates per second; frac = achieved / peak
        assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
        assert set(r["hbm"]) >= {"achieved", "peak", "frac", "frac_vs_8TBs", "unit"}
        assert r["hbm"]["unit"] == "GB/s"


def test_pooled_route_is_hbm_bound():
    r = _roof(3)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["floors_ms_per_step"]["hbm"] > r["floors_ms_per_step"]["sfu"]
    assert abs(r["frac"] - r["achieved"] / HBM) < 1e-3
    assert "sfu" in r and "fp32" in r


def test_floors_match_the_workload_arithmetic():
    # Vim-Small: 64 images x 2 directions x 4097 steps x 768 channels x 16 states
    r = _roof(4)
    upd = 64 * 2 * 4097 * 768 * 16
    assert abs(r["floors_ms_per_step"]["sfu"] - 1e3 * upd / (16 * 148 * SM_MAX * 1e6)) < 1e-4
    # at 3.09 ms per step the SFU fraction is the floor over the time, for any step count
    for steps in (1, 20):
        r = _roof(4, ms=3.09, steps=steps)
        assert abs(r["frac"] - r["floors_ms_per_step"]["sfu"] / 3.09) < 1e-3


def test_backward_lines_stay_on_hbm():
    r = _roof(2, backward=True)
    assert r["bound"] == "hbm" and "sfu" in r
