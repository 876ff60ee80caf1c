"""Host-side arithmetic of bench.py checked on the CPU: the effective-FLOP counts against their closed
forms, the union-tile useful fraction on hand-made masks, the schedule statistics on a synthetic
per-CTA record, the clock sampler's verdict on a recorded CSV, and the DRAM records' binding to the
kernel sources they were captured with."""
import json
import os
import sys
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_effective_flops_matches_the_metric_formula():
    # 4 N^2 d H (1 - sparsity) for the exact pairs plus 4 d 64 per unselected (query block, key
    # block) pair and query token: one pooled key per unselected block
    B, N, H, d = 1, 65536, 32, 128
    Nb = N // 64
    total = B * H * Nb * Nb
    exact = total // 10
    flops, exact_flops = bench.effective_flops(B, N, H, exact, total, d)
    assert exact_flops == pytest.approx(4.0 * N * N * d * H * exact / total, rel=1e-12)
    assert flops - exact_flops == pytest.approx(4.0 * d * 64 * (total - exact), rel=1e-12)


def test_sol2_flops_closed_form():
    B, N, H, d = 1, 65536, 32, 128
    Nb = N // 64
    total, exact = B * H * Nb * Nb, 1000
    f = bench.sol2_flops(B, N, H, exact, total, d)
    tail = 12.0 * d * 2 * (total - exact)          # two 32-token anchors per 64-token block
    corr = 2.0 * d * B * H * N
    assert f == pytest.approx(4.0 * d * 64 * 64 * exact + tail + corr, rel=1e-12)


def test_union_useful_fraction_by_hand():
    # query blocks 0 and 1 form one unit: exact sets {0, 1} and {1, 2}; union of 3 key blocks
    # for 2 rows = 6 computed, 4 useful
    m = np.zeros((1, 1, 3, 3), dtype=bool)
    m[0, 0, 0, [0, 1]] = True
    m[0, 0, 1, [1, 2]] = True
    # query block 2 is alone in its unit (odd count): {2} computed once
    m[0, 0, 2, 2] = True
    assert bench.union_useful_fraction(m) == pytest.approx((4 + 1) / (6 + 1))
    # identical exact sets waste nothing
    m2 = np.ones((1, 2, 4, 4), dtype=bool)
    assert bench.union_useful_fraction(m2) == 1.0


def test_scheduler_stats_on_a_synthetic_schedule(monkeypatch):
    import torch

    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    # two SMs: SM 0 runs units [0, 10) and [10, 20); SM 1 runs [0, 12) and [12, 30) (ns)
    ut = np.array([[0, 10, 0], [10, 20, 0], [0, 12, 1], [12, 30, 1]], dtype=np.int64)
    calls = []
    sa = types.SimpleNamespace(set_unit_timing=lambda on: calls.append(on), last_unit_times=lambda: ut)
    st = bench.scheduler_stats(sa, lambda: None)
    assert calls == [True, False]
    assert st["units"] == 4 and st["sms"] == 2
    assert st["span_ms"] == pytest.approx(30e-6)
    # finishes 20 and 30, median 25: tail (30 - 25) / 30
    assert st["tail_frac"] == pytest.approx(5 / 30)
    assert st["busy_frac"] == pytest.approx((10 + 10 + 12 + 18) / (30 * 2))
    assert st["unit_ms_max"] == pytest.approx(18e-6)


def _sampler_with(tmp_path, lines):
    path = tmp_path / "clocks.csv"
    path.write_text("".join(l + "\n" for l in lines))
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.path = str(path)
    s.fh = open(os.devnull, "w")
    s.proc = types.SimpleNamespace(terminate=lambda: None, wait=lambda timeout=None: 0, kill=lambda: None)
    return s


def test_clock_sampler_reports_the_loaded_median_and_active_reasons(tmp_path):
    row = "0, {sm}, 1965, 900.0, {util}, 0x0, Not Active, Not Active, Not Active, {cap}"
    lines = [row.format(sm=1965, util=0, cap="Not Active"),           # idle sample: left out
             row.format(sm=1845, util=100, cap="Active"),
             row.format(sm=1875, util=100, cap="Not Active"),
             row.format(sm=1905, util=100, cap="Active"),
             "garbage line"]
    out = _sampler_with(tmp_path, lines).stop()
    assert out["sm_mhz"] == 1875 and out["sm_max_mhz"] == 1965 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"]
    hot = _sampler_with(tmp_path, ["0, 1500, 1965, 900.0, 100, 0x0, Not Active, Active, Not Active, Not Active"]).stop()
    assert hot["reasons"] == ["hw_thermal_slowdown"]
    empty = _sampler_with(tmp_path, []).stop()
    assert empty["samples"] == 0 and empty["sm_mhz"] is None


@pytest.mark.parametrize("precision", ["bf16", "fp8"])
def test_committed_dram_records_belong_to_the_committed_kernel_sources(precision, tmp_path, monkeypatch):
    record, source = bench.TRAFFIC[precision]
    with open(record) as f:
        rec = json.load(f)
    for name in ("s32k_90", "s64k"):
        assert bench.measured_traffic(name, precision) == rec[name]["dram_bytes_per_launch"]
    assert bench.measured_traffic("no_such_workload", precision) is None
    # a source that differs from the captured one yields no traffic figure
    other = tmp_path / "kernel.cu"
    other.write_text(open(source).read() + "\n// changed\n")
    monkeypatch.setitem(bench.TRAFFIC, precision, (record, str(other)))
    assert bench.measured_traffic("s64k", precision) is None
