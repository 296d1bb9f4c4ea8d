"""The benchmark's host-side accounting (CPU only): the algorithmic bytes and FLOPs behind the
roofline fractions, the stored ncu traffic figure and when it applies, the peaks, and the
throughput arithmetic."""
import json
import os

import numpy as np
import pytest

import bench
from workloads import BEAM, TINY

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_per_unit_figures_of_the_beam_layer():
    """Per expert hit: gate + up + down codes and E4M3 scales at 0.5625 bytes per value
    (3 * 2560 * 5120 values = 22,118,400 bytes) plus four FP32 global scales; per token:
    2 * 8 * 3 * H * I = 629,145,600 FP4 FLOPs."""
    counts = np.zeros(BEAM.E, dtype=np.int64)
    counts[:3] = [1, 0, 2]
    counts[5] = 7
    a1 = bench.algorithmic(BEAM, 1, counts)
    a2 = bench.algorithmic(BEAM, 2, counts)
    assert a1["experts_hit"] == 3
    per_token_flops = 2 * 8 * 3 * BEAM.H * BEAM.I
    assert per_token_flops == 629_145_600
    assert a1["flops"] == per_token_flops and a2["flops"] == 2 * per_token_flops
    # the layer's bytes: weights of the experts hit, BF16 in and out, the FP32 router
    weights = 3 * (3 * BEAM.I * BEAM.H * 9 // 16 + 16)
    assert 3 * BEAM.I * BEAM.H * 9 // 16 + 16 == 22_118_416
    assert a1["layer_bytes"] == weights + 1 * BEAM.H * 4 + BEAM.E * BEAM.H * 4
    # gate/up: its weights (2/3 of the codes and scales, two globals), gathered A rows, h rows
    gu = 3 * (2 * BEAM.I * BEAM.H * 9 // 16 + 8) + 8 * BEAM.H * 9 // 16 + 8 * BEAM.I * 9 // 16
    assert a1["gateup_bytes"] == gu
    assert a1["gateup_flops"] == 2 * 8 * 2 * BEAM.I * BEAM.H


def test_decode_step_bytes_match_the_stated_figure():
    """99 experts hit at T = 16 move 2.20 GB per step, the figure the measurements quote."""
    counts = np.zeros(BEAM.E, dtype=np.int64)
    counts[:99] = 1
    b = bench.algorithmic(BEAM, 16, counts)["layer_bytes"]
    assert abs(b / 1e9 - 2.20) < 0.005


def test_stored_traffic_applies_only_to_its_sources_and_workload(monkeypatch):
    t = bench.stored_traffic("decode", 99)
    with open(os.path.join(ROOT, "profiles", "gemm_gateup_traffic.txt")) as f:
        vals = dict(line.split()[:2] for line in f if line.strip() and not line.startswith("#"))
    assert vals["source_sha256"] == bench.kernel_source_hash()
    assert t == float(vals["dram_bytes_per_launch"]) / float(vals["experts_hit"]) * 99
    assert bench.stored_traffic("prefill", 99) is None
    assert bench.stored_traffic("decode", 50) == t * 50 / 99
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 64)
    assert bench.stored_traffic("decode", 99) is None


def test_peaks_are_the_measured_file_else_the_fallback():
    p = bench.peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
        return
    with open(path) as f:
        m = json.load(f)
    assert p["source"] == "measured" and p["hbm_gbs"] == m["hbm_gbs"] and p["bf16_tflops"] == m["bf16_tflops"]


def test_throughput_is_all_ranks_tokens_over_the_slowest_rank():
    assert bench.tokens_per_second(1, 16, 500, 181.8) == pytest.approx(16 * 500 / 0.1818, rel=1e-12)
    assert bench.tokens_per_second(4, 16, 100, 40.0) == pytest.approx(4 * 16 * 100 / 0.040, rel=1e-12)
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_small_layer_accounting_scales_with_the_shape():
    counts = np.ones(TINY.E, dtype=np.int64)
    a = bench.algorithmic(TINY, 4, counts)
    assert a["experts_hit"] == TINY.E
    assert a["flops"] == 2 * 4 * TINY.topk * 3 * TINY.H * TINY.I
