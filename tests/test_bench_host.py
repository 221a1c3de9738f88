"""Host logic of bench.py that its reported numbers rest on, checked on the
CPU: the algorithmic bytes of a bf16 layer (the roofline's numerator), the
whole-job per-layer time, and the clock-record parsing that decides whether
a run is kept (throttle reasons, median SM clock)."""
import numpy as np

import bench


def test_layer_alg_counts_touched_experts_once():
    H, F, K = 128, 256, 4
    idx = np.array([[0, 1, 1, 5], [5, -1, 0, 7]], dtype=np.int32)   # experts 0, 1, 5, 7
    a = bench.layer_alg(idx, 2, H, F, K)
    assert a["touched_experts"] == 4
    weights = 4 * (2 * F * H + H * F) * 2        # gate_up [2F,H] + down [H,F], bf16
    io = 2 * H * 2 * 2 + 2 * K * (4 + 4)          # x and out (bf16), ids and weights (4 B each)
    assert a["bytes"] == weights + io
    assert a["flops"] == 2 * 2 * K * (2 * F * H + H * F)


def test_per_layer_us_is_whole_job():
    # 4 ranks, 10 steps each, the slowest rank took 800 us in all
    assert bench.per_layer_us(800.0, 10, 4) == 20.0
    assert bench.per_layer_us(800.0, 10, 1) == 80.0


def _summary(lines):
    c = bench.ClockSampler(0)
    c.out = "\n".join(lines)
    return c.summary()


def test_clock_summary_reasons_and_median():
    s = _summary(["1965, 1965, 700.1, Not Active, Not Active, Not Active, Not Active",
                  "1950, 1965, 900.0, Not Active, Not Active, Not Active, Active",
                  "1965, 1965, 950.2, Not Active, Not Active, Not Active, Active"])
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    s = _summary(["1200, 1965, 500.0, Active, Not Active, Active, Not Active"])
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert _summary([])["reasons"] == ["nvidia-smi unavailable"]
