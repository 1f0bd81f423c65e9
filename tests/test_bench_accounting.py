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


def test_fp4_bytes():
    # codes (out + B) in/2, scale bytes (out + B) in/block, y bf16
    assert bench.fp4_bytes(8192, 28672, "nvfp4", 16) == (8192 + 16) * (14336 + 1792) + 16 * 8192 * 2
    assert bench.fp4_bytes(8192, 28672, "mxfp4", 1) == 8193 * (14336 + 896) + 8192 * 2


def test_layer_plan_groups_qkv_and_gate_up():
    class W:
        def __init__(self, name, inn):
            self.name, self.in_features = name, inn

    mats = [(n, W(n, i)) for _ in range(2) for n, (o, i) in wl.LLAMA3_8B.items()]
    xs = {4096: "x4096", 14336: "x14336"}
    ys = {n: "y_" + n for n in wl.LLAMA3_8B}
    plan = bench.layer_plan(mats, xs, ys)
    assert len(plan) == 8
    assert [[w.name for w in p[0]] for p in plan[:4]] == [
        ["q_proj", "k_proj", "v_proj"], ["o_proj"], ["gate_proj", "up_proj"], ["down_proj"]]
    assert [p[1] for p in plan[:4]] == [["y_q_proj", "y_k_proj", "y_v_proj"], ["y_o_proj"],
                                        ["y_gate_proj", "y_up_proj"], ["y_down_proj"]]
    assert plan[0][2] == "x4096" and plan[3][2] == "x14336"
    # the second layer's products, not the first one's again
    assert plan[4][0][0] is mats[7][1] and plan[7][0][0] is mats[13][1]
