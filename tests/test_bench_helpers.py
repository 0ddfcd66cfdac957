"""The measurement arithmetic of bench.py, on the CPU: algorithmic bytes, peaks, throughput, the L2 flush
policy, the clock summary and the command line.

The byte counts are checked against the layer's definition (each touched expert's gate, up and down
matrices read once, W_r, x in, out), written out here with the workload sizes; the clock summary against a
hand-made sample list (NVML's reason bits).
"""
import importlib.util
import json
import os

import pytest

from prefill_sigmoid_top_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_bytes_decode(bench):
    cfg = inputs.WORKLOADS[1]  # M=8, H=7168, I=2048, E=256, top_k=16
    ab = bench.algorithmic_bytes(cfg, touched=95)
    expert = 3 * 2048 * 7168 * 2  # 88.08 MB of bf16 weights per touched expert
    assert expert == 88_080_384
    assert ab["layer"] == 95 * expert + 256 * 7168 * 2 + 2 * 8 * 7168 * 2
    assert ab["layer"] == 8_371_535_872  # the figure the decode bench line reports
    assert ab["up"] == 95 * 2 * 2048 * 7168 * 2 + 8 * 7168 * 2
    assert ab["down"] == 95 * 2048 * 7168 * 2
    assert ab["finalize"] == 8 * 16 * 7168 * 2 + 2 * 8 * 7168 * 2


def test_algorithmic_bytes_nvfp4(bench):
    cfg = inputs.WORKLOADS[4]
    ab = bench.algorithmic_bytes(cfg, touched=256, nvfp4=True)
    # e2m1: half a byte per element, plus one e4m3 scale per 16 elements
    per_expert = 3 * 2048 * 7168 * (0.5 + 1 / 16)
    assert ab["layer"] == int(256 * per_expert + 256 * 7168 * 2 + 2 * 1000 * 7168 * 2)
    assert abs(256 * per_expert / 1e9 - 6.342) < 1e-3  # 6.34 GB of prepared weights


def test_aggregate_is_all_ranks_over_the_slowest(bench):
    assert bench.aggregate(8 * 20, 0.025, 1) == pytest.approx(6400.0)
    assert bench.aggregate(8 * 20, 0.025, 4) == pytest.approx(25600.0)
    assert bench.reduce_max(1.5, 1) == 1.5


def test_peaks_are_the_measured_ones(bench):
    hbm, tc, kind = bench.peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        assert (hbm, tc, kind) == (float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured")
    else:
        assert (hbm, tc, kind) == (6650.0, 1590.0, "fallback")


def test_l2_flush_policy(bench):
    # a step flushes L2 when the layer's bytes fit in L2 a few times over (the tiny workload), not otherwise
    tiny = bench.algorithmic_bytes(inputs.WORKLOADS[0], touched=8)["layer"]
    decode = bench.algorithmic_bytes(inputs.WORKLOADS[1], touched=95)["layer"]
    assert tiny < 4 * 126_000_000 <= decode


def test_clock_summary_reasons_and_median(bench):
    cs = bench.ClockSampler(0)
    cs.max_mhz = 1965.0
    cs.samples = [(1965.0, 0x0), (1900.0, 0x4), (1800.0, 0x4 | 0x20), (1965.0, 0x0), (1940.0, 0x0)]
    s = cs.summary()
    assert s["sm_mhz"] == 1940.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 5
    assert s["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    empty = bench.ClockSampler(0)
    assert empty.summary() is None
    empty.error = "no NVML"
    assert empty.summary() == {"error": "no NVML"}


def test_command_line_defaults(bench):
    a = bench.parse_args([])
    assert (a.gpus, a.steps, a.warmup, a.config, a.impl) == (1, 20, 3, 1, "ours")
    assert not a.route_only and not a.no_cpu_baseline
    a = bench.parse_args(["--config", "3", "--route-only", "--steps", "5"])
    assert a.config == 3 and a.route_only and a.steps == 5
    w = bench.workload(bench.parse_args(["--config", "1", "--experts", "32"]))
    assert (w.M, w.E, w.K) == (8, 32, 16) and w.name == "decode_m8_E32"


def test_default_run_measures_all_four_workloads(bench):
    assert bench.workload_list(bench.parse_args([])) == [1, 2, 3, 4]
    assert bench.workload_list(bench.parse_args(["--config", "3"])) == [3]
    assert bench.workload_list(bench.parse_args(["--experts", "32"])) == [1]  # a smaller copy: headline only
    assert bench.workload_list(bench.parse_args(["--config", "0", "--workloads", "all"])) == [0, 1, 2, 3, 4]
    assert bench.workload_list(bench.parse_args(["--workloads", "none"])) == [1]


def test_layer_roofline_fractions(bench):
    # prefill: 2 * 3 * H * I * M * K flops; graded on the bf16 tensor peak, HBM fraction beside it
    cfg = inputs.WORKLOADS[3]
    r = bench.layer_roofline(cfg, 256, 0.004, 6541.5, 1617.9, read_ceiling=7200.0)
    flops = 2 * 3 * 7168 * 2048 * 2048 * 16
    assert r["tflops"] == pytest.approx(flops / 0.004 / 1e12)
    assert r["bound"] == "tensor" and r["frac"] == r["frac_tensor"] == pytest.approx(r["tflops"] / 1617.9)
    ab = 256 * 88_080_384 + 256 * 7168 * 2 + 2 * 2048 * 7168 * 2
    assert r["algorithmic_bytes"] == ab and r["frac_hbm"] == pytest.approx(ab / 0.004 / 1e9 / 6541.5)
    assert r["frac_read_ceiling"] == pytest.approx(ab / 0.004 / 1e9 / 7200.0)
    # NVFP4: HBM-graded; the tensor peak is the measured bf16 peak x 4 (nominal fp4 / bf16)
    r4 = bench.layer_roofline(inputs.WORKLOADS[4], 256, 0.0015, 6541.5, 1617.9)
    assert r4["bound"] == "hbm" and r4["tensor_peak_tflops"] == pytest.approx(4 * 1617.9)
    assert bench.layer_roofline(inputs.WORKLOADS[1], 95, 0.0012, 6541.5, 1617.9)["bound"] == "hbm"
    assert bench.layer_roofline(inputs.WORKLOADS[2], 256, 0.0036, 6541.5, 1617.9)["bound"] == "hbm"
