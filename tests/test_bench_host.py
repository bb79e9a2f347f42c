"""Host-side logic of bench.py that decides what the JSON line reports: the clock
samples it keeps, the algorithmic work per launch behind the roofline, and the
DRAM-traffic record lookup (no GPU needed)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _line(uuid, sm, smax, power_cap="Not Active", hw="Not Active"):
    return f"{uuid}, {sm}, {smax}, 900.0, 0x0, {hw}, Not Active, Not Active, {power_cap}"


def test_clock_summary_keeps_only_the_region_and_this_gpu():
    s = bench.ClockSampler("GPU-abc")
    s.lines = [_line("GPU-abc", 1965, 1965),                    # before the region: dropped
               _line("GPU-abc", 1700, 1965, power_cap="Active"),
               _line("GPU-other", 900, 1965, hw="Active"),       # another GPU: ignored
               "garbage line",
               _line("GPU-abc", 1720, 1965),
               _line("GPU-abc", 1690, 1965)]
    s.first = 1
    out = s.summary()
    assert out["samples"] == 3
    assert out["sm_mhz"] == pytest.approx(1700.0)
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_samples_says_so():
    s = bench.ClockSampler("GPU-abc")
    s.lines = [_line("GPU-abc", 1965, 1965)]
    s.first = 1
    out = s.summary()
    assert out["samples"] == 0 and out["sm_mhz"] is None and out["reasons"] == ["clocks not sampled"]


def test_work_per_launch_matches_the_shapes():
    B, ni, nt = 1, 4096, 256
    N, D, F = ni + nt, 1536, 4096
    assert bench.kernel_work("attention", B, ni, nt) == ("flop", 4.0 * N * N * D)
    assert bench.kernel_work("gemm_qkv", B, ni, nt) == ("flop", 2.0 * N * D * 3 * D)
    assert bench.kernel_work("gemm_w13", 2, ni, nt) == ("flop", 2.0 * 2 * N * D * 2 * F)
    assert bench.kernel_work("rmsnorm_mod", B, ni, nt) == ("byte", N * D * 6.0)
    # one 48-block forward: the per-block GEMMs and attention, plus the input and output heads
    per_block = 2 * N * D * (3 * D + D + 2 * F + F) + 4 * N * N * D
    heads = 2 * nt * 4 * 2880 * D + 2 * ni * 128 * D * 2
    assert bench.forward_flops(ni, nt) == 48 * per_block + heads
    assert bench.forward_flops(ni, nt) == pytest.approx(17.43e12, rel=5e-3)   # the 1024^2 forward


def test_traffic_record_lookup():
    assert bench.dram_traffic("attention", "no_such_workload") is None
    assert bench.dram_traffic("gemm_out", "turbo_1024") is None          # no record for that kernel
    got = bench.dram_traffic("attention", "turbo_1024")
    assert got is None or 3.0e7 < got < 6.0e7                             # q, k, v read once when current
