"""Host logic of bench.py on CPU: the roofline arithmetic (HBM and L2 bases, bound time),
the timed-region repeats, and the reference arm (the CPU oracle) end to end."""
import json
import os
import subprocess
import sys

import pytest

import bench
import workloads

W = workloads.WORKLOADS


def fake_peaks(gather_xpair=450.0, red_xpair=300.0, red_f16_xpair=320.0):
    def rates(x):
        return {w: {"random": 100.0, "xpair": x} for w in ("4", "8", "16")}
    b = {"gather": rates(gather_xpair), "red": rates(red_xpair), "red_f16": rates(red_f16_xpair)}
    return {"buffers": {"32MiB": b, "64MiB": b}}


def test_roofline_hbm_basis(monkeypatch):
    monkeypatch.setattr(bench, "measured_peaks", lambda: (5000.0, "test"))
    n, ms = 1 << 18, 0.1
    r = bench.roofline(W["grid_L16F2T19"], "fwd", n, ms, "forward_kernel", None)
    alg = 1164 * n
    assert r["bound"] == "hbm" and r["algorithmic_bytes_per_launch"] == alg
    assert r["achieved"] == pytest.approx(alg / (ms * 1e-3) / 1e9, rel=1e-3)
    assert r["frac"] == pytest.approx(alg / (ms * 1e-3) / 1e9 / 5000.0, rel=1e-3)
    assert "l2" not in r
    # without L2 peaks the bound time is the HBM time of the streams (x + output rows)
    assert r["bound_time_ms"] == pytest.approx((12 + 128) * n / 5000e9 * 1e3, rel=1e-3)


def test_roofline_l2_basis(monkeypatch):
    monkeypatch.setattr(bench, "measured_peaks", lambda: (5000.0, "test"))
    n, ms = 1 << 18, 0.1
    r = bench.roofline(W["grid_L16F2T19"], "fwd", n, ms, "forward_kernel", fake_peaks(gather_xpair=450.0))
    ops = 8 * 16 * n                                   # 8 corners x 16 levels per point
    assert r["l2"]["ops_per_launch"] == ops
    assert r["l2"]["frac"] == pytest.approx(ops / 450e9 / (ms * 1e-3), rel=1e-3)
    assert r["l2"]["frac_vs_random_units"] == pytest.approx(ops / 100e9 / (ms * 1e-3), rel=1e-3)
    assert r["bound_by"] == "l2" and r["frac_bound_time"] == r["l2"]["frac"]
    # backward: 8-byte fp32 reductions (F = 2) against the reduction probe
    b = bench.roofline(W["rays_L16F2T19"], "bwd", 1 << 20, 0.35, "backward_kernel", fake_peaks(red_xpair=300.0))
    assert "8-byte f32" in b["l2"]["access"]
    assert b["l2"]["frac"] == pytest.approx(8 * 16 * (1 << 20) / 300e9 / 0.35e-3, rel=1e-3)
    # fp16 gradient: 4-byte fp16 reductions, their own probe and algorithmic bytes
    h = bench.roofline(W["rays_L16F2T19"], "bwd", 1 << 20, 0.32, "backward_kernel_half", fake_peaks(), grad_dtype="f16")
    assert "4-byte f16" in h["l2"]["access"] and h["l2"]["peak_g_ops_per_s"] == 320.0
    assert h["algorithmic_bytes_per_launch"] == (12 + 128 + 8 * 32 * 2) * (1 << 20)


def test_roofline_reduction_requests(monkeypatch):
    """The backward's L2 reduction requests (an ncu count) against the random-unit
    reduction rate of the same width: one request per operation."""
    monkeypatch.setattr(bench, "measured_peaks", lambda: (5000.0, "test"))
    monkeypatch.setattr(bench, "ncu_entry", lambda k, w: {"l2_red_requests_per_launch": 55e6, "dram_bytes_per_launch": 1e8})
    b = bench.roofline(W["rays_L16F2T19"], "bwd", 1 << 20, 0.35, "backward_kernel", fake_peaks())
    rr = b["l2_red_requests"]
    assert rr["per_launch"] == 55_000_000 and rr["g_per_s"] == pytest.approx(55e6 / 0.35e-3 / 1e9, abs=0.05)
    assert rr["peak_g_per_s"] == 100.0 and rr["frac"] == pytest.approx(55e6 / 0.35e-3 / 100e9, rel=1e-3)
    assert "random 8-byte" in rr["peak_source"]
    # without probe peaks only the count and rate are reported
    assert "frac" not in bench.roofline(W["rays_L16F2T19"], "bwd", 1 << 20, 0.35, "backward_kernel", None)["l2_red_requests"]


def test_roofline_large_grid_is_hbm_bound_per_level(monkeypatch):
    """The 1 GiB table does not fit in L2: every algorithmic byte crosses HBM, and the L2
    term uses one level's 64 MB slice (the level-major schedule's working set)."""
    monkeypatch.setattr(bench, "measured_peaks", lambda: (5000.0, "test"))
    n, ms = 1 << 22, 2.8
    r = bench.roofline(W["large_L16F4T22"], "fwd", n, ms, "forward_kernel", fake_peaks(gather_xpair=1e6))
    assert r["bound_by"] == "hbm"
    assert r["bound_time_ms"] == pytest.approx(2316 * n / 5000e9 * 1e3, rel=1e-3)
    assert "64MiB" in r["l2"]["peak_source"] and "16-byte" in r["l2"]["access"]


def test_roofline_level_major_schedule(monkeypatch):
    """A table that fits in L2, run level by level: the L2 term uses one level's slice
    (4 MB for the default grid, the 32 MiB probe buffer), and the HBM term only the
    streams, as for the point-major forward."""
    monkeypatch.setattr(bench, "measured_peaks", lambda: (5000.0, "test"))
    n, ms = 1 << 18, 0.095
    r = bench.roofline(W["grid_L16F2T19"], "fwd", n, ms, "forward_kernel_levels", fake_peaks(), level_major=True)
    assert "32MiB" in r["l2"]["peak_source"] and r["bound_by"] == "l2"
    p = bench.roofline(W["grid_L16F2T19"], "fwd", n, ms, "forward_kernel", fake_peaks())
    assert "64MiB" in p["l2"]["peak_source"] and r["frac"] == p["frac"]


def test_loop_repeats_reach_the_minimum_timed_region():
    for steps, step_s in [(20, 0.7e-3), (3, 5e-3), (50, 1e-4)]:
        r = bench.loop_repeats(steps, step_s, 1.0)
        assert r * steps * step_s >= 1.0 and (r - 1) * steps * step_s < 1.0


@pytest.mark.timeout(300)
def test_reference_arm_prints_one_line():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_L4F2T10", "--steps",
                        "1", "--warmup", "1"], cwd=root, env=env, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
