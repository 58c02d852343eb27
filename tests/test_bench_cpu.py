"""bench.py on the CPU: its pieces exist and its host-side arithmetic and
argument handling behave (the timed paths themselves need a GPU)."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_entry_points_exist():
    for name in ("Problem", "ClockSampler", "time_device", "time_e2e", "cpu_baseline", "extra_workloads",
                 "head_workloads", "time_head", "head_line", "run_native", "run_head", "run_reference", "main",
                 "measured_peaks", "recorded_traffic", "kernel_source_hash"):
        assert callable(getattr(bench, name, None)), name


def test_aggregate_throughput_and_peaks():
    assert bench.aggregate_throughput(1000, 2, 4, 8.0) == 1000 * 2 * 4 / 8e-3
    p = bench.measured_peaks()
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    assert len(bench.kernel_source_hash()) == 16


def test_head_line_arithmetic():
    from nonlinear_rnn_iteration_b200 import workloads

    w = workloads.HEAD_WORKLOADS["headgru_8x4096x512_h8_k3"]
    line = bench.head_line(w, 10.0, 5.0, "PARARNN_OK")
    useful = 2.0 * 64 ** 3 * 8 * 4096 * 8 * 3 / 1e-2 / 1e12
    assert abs(line["roofline"]["achieved_useful"] - round(useful, 2)) < 1e-9
    assert line["elem_per_s"] == w.elements / 1e-2
    assert line["bwd_elem_per_s"] == w.elements / 5e-3
    json.dumps(line)


def test_help_lists_every_workload():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], capture_output=True, text=True,
                         cwd=ROOT, check=True).stdout
    for name in ("linear_8x16384x1024", "gru_1x131072x4096_k2_bf16", "headgru_8x4096x512_h8_k3"):
        assert name in out


def test_streaming_bytes_per_element():
    # one HBM pass per Newton iteration: the first reads px and writes the
    # state, each later one also reads the state back
    from nonlinear_rnn_iteration_b200 import workloads

    W = workloads.WORKLOADS
    assert bench.streaming_bytes_per_elem(W["linear_8x16384x1024"], "fwd") == 12
    assert bench.streaming_bytes_per_elem(W["gru_8x4096x2048_k3"], "fwd") == 16 + 20 + 20
    assert bench.streaming_bytes_per_elem(W["gru_8x4096x2048_k3_bf16"], "fwd") == 10 + 14 + 14
    assert bench.streaming_bytes_per_elem(W["lstm_4x32768x1024_k4"], "fwd") == 24 + 3 * 32
    assert bench.streaming_bytes_per_elem(W["gru_1x131072x4096_k2_bf16"], "fwd") == 10 + 14
    assert bench.streaming_bytes_per_elem(W["gru_1x131072x4096_k2_bf16"], "bwd") == 26
    w = W["gru_1x131072x4096_k2_bf16"]
    r = bench.kernel_roofline(w, "fwd", 2.0, {"hbm_gbs": 6000.0, "source": "of test"})
    assert r["algorithmic_bytes_per_launch"] == 24 * w.elements
    assert abs(r["achieved"] - round(24 * w.elements / 2e-3 / 1e9, 1)) < 1e-9
    assert r["frac"] == round(r["achieved"] / 6000.0, 4)
    assert r["fused_bytes_per_elem"] == 10
    json.dumps(r)
