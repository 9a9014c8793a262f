"""Host-side pieces of bench.py that the reported numbers rest on: algorithmic bytes per
workload (the roofline's numerator for HBM-bound lines), the launch count per step, the peak
table and the rule that a DRAM-traffic record only counts for the kernel source it was taken
on.  No GPU."""
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


# Bytes = A + B read once, C written, C read again when beta != 0 (the definition the
# roofline uses); values in MB as 1e6 bytes.
EXPECTED_MB = {
    "square256": 0.524288,        # 2 x 256^2 bf16 + 256^2 fp32
    "square8192": 402.653184,
    "edge4099": 134.414408,       # beta = 1: C read and written
    "edge8192x256": 77.594624,
    "recsys": 402.915328,         # W once, X and Y per batch entry
}


@pytest.mark.parametrize("name", sorted(EXPECTED_MB))
def test_algorithmic_bytes(name):
    assert bench.algorithmic_bytes(bench.WORKLOADS[name]) / 1e6 == pytest.approx(EXPECTED_MB[name],
                                                                                  abs=1e-6)


def test_algorithmic_bytes_thin_edge():
    # 127x8191x2048: A 127*2048*2 + B 8191*2048*2 + C read and written 2 * 127*8191*2
    w = bench.WORKLOADS["edge127x8191"]
    assert bench.algorithmic_bytes(w) == 127 * 2048 * 2 + 8191 * 2048 * 2 + 2 * 127 * 8191 * 2


def test_roofline_bound_follows_the_ridge():
    peaks = {"bf16_tflops": 1698.2, "hbm_gbs": 6457.1}
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    for name, w in bench.WORKLOADS.items():
        _, batch, M, N, K, *_ = w
        intensity = bench.executed_flops(w) / bench.algorithmic_bytes(w)
        # square and LLM shapes and 4099^3 above the ridge; the thin edges and RecSys below
        expect_tensor = name in ("square4096", "square8192", "llm_up", "llm_down", "edge4099",
                                 "square4096_f16", "square8192_f16")
        assert (intensity >= ridge) == expect_tensor, (name, intensity, ridge)


def test_launches_per_step():
    assert bench.launches_per_step(bench.WORKLOADS["edge4099"]) == 3  # two pre-pass copies
    for name in ("square8192", "edge8192x256", "edge127x8191", "recsys", "square256"):
        assert bench.launches_per_step(bench.WORKLOADS[name]) == 1, name


def test_traffic_record_needs_matching_kernel_source(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["square8192"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["kernel_source_hash"])
    assert bench.recorded_traffic("square8192") == float(rec["dram_bytes_per_launch"])
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("square8192") is None
    assert bench.recorded_traffic("no-such-workload") is None


def test_peaks_fall_back_when_unmeasured(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback"
    assert peaks["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]


def test_default_workload_is_the_headline_config():
    assert bench.DEFAULT_WORKLOAD == "square8192"
    _, batch, M, N, K, out, alpha, beta, *_ = bench.WORKLOADS["square8192"]
    assert (batch, M, N, K, out, alpha, beta) == (1, 8192, 8192, 8192, "bf16", 1.0, 0.0)


def test_l2_flush_rule():
    """Workloads whose data are under twice the L2 cache are timed cold (flushed); the others
    run back to back."""
    flushed = sorted(n for n, w in bench.WORKLOADS.items() if bench.needs_flush(w))
    assert flushed == ["edge127x8191", "edge4099", "edge8192x256", "recsys_dedup128", "recsys_dedup4",
                       "square256", "square4096", "square4096_f16"]


def test_fp16_workloads_use_fp16_operands():
    for name in ("square8192_f16", "square4096_f16"):
        w = bench.WORKLOADS[name]
        assert w.in_dtype == "f16" and w.out == "f16"
    assert all(w.in_dtype == "bf16" for n, w in bench.WORKLOADS.items() if not n.endswith("_f16"))


def test_dedup_workloads():
    w = bench.WORKLOADS["recsys_dedup128"]
    idx = bench.dedup_index(w)
    assert idx.shape == (2048,) and idx.min() == 0 and idx.max() == 15
    assert np.all(np.bincount(idx) == 128)  # 16 requests of 128 items
    assert np.all(np.bincount(bench.dedup_index(bench.WORKLOADS["recsys_dedup4"])) == 4)
    # X is read once per distinct entry; Y is written per item; the index is read once
    assert bench.algorithmic_bytes(w) == 256 * 512 * 2 + 16 * 512 * 128 * 2 + 2048 * 256 * 128 * 2 + 2048 * 4
    assert bench.executed_flops(w) == 2.0 * 16 * 256 * 128 * 512
    assert bench.launches_per_step(w) == 2
