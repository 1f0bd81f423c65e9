"""The bench's byte accounting, clock-sample parsing and peak lookup, on the
CPU: the algorithmic bytes behind every GB/s and roofline fraction it prints
are the formulas stated for them, at the layer shapes the bench uses."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from post_weight_quantization_group_b200 import workloads as wl  # noqa: E402


def test_w4a16_bytes_70b_down():
    # codes out*in/2 + fp16 scales out*(in/128)*2 + x B*in*2 + y B*out*2
    assert bench.algo_bytes(8192, 28672, 128, 1) == 117_440_512 + 3_670_016 + 57_344 + 16_384
    assert bench.algo_bytes(8192, 28672, 64, 1, sym=False) == (117_440_512 + 2 * 7_340_032
                                                                + 57_344 + 16_384)


def test_8b_step_bytes():
    layer = sum(bench.algo_bytes(o, i, 128, 1) for o, i in wl.LLAMA3_8B.values())
    assert layer == pytest.approx(112.6e6, rel=1e-3)
    # the default bench line's bytes_per_step: 32 distinct layers
    assert 32 * layer == 3_603_955_712
    # the fused q/k/v + gate/up layout reads x three fewer times per layer
    fused = sum(bench.algo_bytes(o, 4096, 128, 1) for o in (6144, 4096, 28672))
    fused += bench.algo_bytes(4096, 14336, 128, 1)
    assert 32 * fused == 3_603_169_280 == 32 * layer - 32 * 3 * 4096 * 2


def test_dense_and_quantizer_bytes():
    assert bench.dense_bytes(8192, 28672, 1) == 8192 * 28672 * 2 + 28672 * 2 + 8192 * 2
    # fp16 in, codes and fp16 scales out
    assert bench.quant_bytes(4096, 4096, 128) == 4096 * 4096 * 2 + 4096 * 2048 + 4096 * 32 * 2


def test_clock_summary_parses_samples_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    c.lines = ["0, 1200, 1965, 500, 0x40, Active, Not Active, Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_peaks_fall_back_without_measurements(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks["hbm_gbs"] == 6650.0
