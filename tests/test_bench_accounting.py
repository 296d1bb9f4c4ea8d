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
    # down: its weights (1/3 of the codes and scales, two globals) and its A operand (the h rows)
    assert a1["down_bytes"] == 3 * (BEAM.I * BEAM.H * 9 // 16 + 8) + 8 * BEAM.I * 9 // 16
    assert a1["down_flops"] == 2 * 8 * BEAM.H * BEAM.I
    assert a1["gateup_flops"] + a1["down_flops"] == a1["flops"]


def test_decode_step_bytes_match_the_stated_figure():
    """99 experts hit at T = 16 move 2.20 GB per step, the figure the measurements quote."""
    counts = np.zeros(BEAM.E, dtype=np.int64)
    counts[:99] = 1
    b = bench.algorithmic(BEAM, 16, counts)["layer_bytes"]
    assert abs(b / 1e9 - 2.20) < 0.005


def test_stored_traffic_applies_only_to_its_sources_and_workload(monkeypatch):
    with open(bench.TRAFFIC_FILE) as f:
        vals = dict(line.split()[:2] for line in f if line.strip() and not line.startswith("#"))
    if vals["source_sha256"] != bench.kernel_source_hash():
        # the kernels changed since the counters were taken: the line reports no traffic
        assert bench.stored_traffic("decode", 99) is None
        assert bench.traffic_note("decode").startswith("none: ") and "hash" in bench.traffic_note("decode")
        monkeypatch.setattr(bench, "kernel_source_hash", lambda: vals["source_sha256"])
    assert "one ncu capture" in bench.traffic_note("decode")
    assert bench.traffic_note("prefill").startswith("none: ")
    t = bench.stored_traffic("decode", 99)
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


def test_prefill_down_bytes_match_the_stated_figure():
    """At T = 4096 with every expert hit the down GEMM moves 1.934 GB: 256 experts x 7,372,808
    bytes of weights plus 32,768 pairs x 1,440 bytes of requantised h."""
    counts = np.full(BEAM.E, 128, dtype=np.int64)
    a = bench.algorithmic(BEAM, 4096, counts)
    assert a["down_bytes"] == 256 * 7_372_808 + 32_768 * 1_440
    assert abs(a["down_bytes"] / 1e9 - 1.9346) < 0.0001


def test_kernel_roofline_takes_the_binding_bound_and_the_burst_fp4_peak():
    p = {"hbm_gbs": 6546.2, "bf16_tflops": 1615.2, "bf16_tflops_sustained": 1365.0, "source": "measured"}
    burst, sustained = bench.fp4_peaks(p)
    assert burst == pytest.approx(6460.8) and sustained == pytest.approx(5460.0)
    # decode gate/up: 1.46 GB, 5.2 GFLOP in 0.2157 ms -> HBM bound
    r = bench.kernel_roofline(1_460_368_152, 5.2e9, 0.2157, p)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(1_460_368_152 / 0.2157e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6546.2)
    assert r["frac_of_spec"] == pytest.approx(r["achieved"] / bench.HBM_SPEC_GBS)
    # T = 32768 gate/up: 13.7 TFLOP in 3.30 ms -> tensor bound, scored against the burst peak
    r = bench.kernel_roofline(6.4e9, 13.74e12, 3.30, p)
    assert r["bound"] == "tensor" and r["peak"] == pytest.approx(burst)
    assert r["frac"] == pytest.approx(13.74e12 / 3.30e-3 / 1e12 / burst)
    assert r["fp4_frac_sustained"] == pytest.approx(13.74e12 / 3.30e-3 / 1e12 / sustained)
    assert r["fp4_frac"] == r["frac"] and r["hbm_frac"] == pytest.approx(6.4e9 / 3.30e-3 / 1e9 / 6546.2)


def test_config_entry_reports_the_dominant_kernel():
    p = {"hbm_gbs": 6546.2, "bf16_tflops": 1615.2, "bf16_tflops_sustained": 1365.0, "source": "measured"}
    counts = np.full(BEAM.E, 1024, dtype=np.int64)
    alg = bench.algorithmic(BEAM, 32768, counts)
    gemms = {"gateup": bench.kernel_roofline(alg["gateup_bytes"], alg["gateup_flops"], 3.3, p),
             "down": bench.kernel_roofline(alg["down_bytes"], alg["down_flops"], 3.3, p)}
    m = {"workload": "w", "T_per_rank": 32768, "experts_hit": 256, "ms_per_step": 8.0, "value": 1.0,
         "stage_ms": {}, "alg": alg, "layer_roofline": {}, "gemms": gemms,
         "dominant": {**gemms["gateup"], "kernel": bench.GATEUP_KERNEL}}
    e = bench.config_entry(m, None)
    assert e["roofline"]["bound"] == "tensor" and e["roofline"]["frac"] == gemms["gateup"]["frac"]
    assert e["roofline"]["kernel"] == bench.GATEUP_KERNEL
    assert e["gemms"]["down"]["bound"] == "tensor"
    # short segments: the one launch that runs both GEMMs, on both GEMMs' bytes
    counts = np.zeros(BEAM.E, dtype=np.int64)
    counts[:99] = 1
    alg = bench.algorithmic(BEAM, 16, counts)
    both = bench.kernel_roofline(alg["gateup_bytes"] + alg["down_bytes"], alg["gateup_flops"] + alg["down_flops"],
                                 0.32, p)
    m.update({"alg": alg, "dominant": {**both, "kernel": bench.EXPERTS_KERNEL}})
    e = bench.config_entry(m, None)
    assert e["roofline"]["bound"] == "hbm" and e["roofline"]["kernel"] == bench.EXPERTS_KERNEL
    assert e["roofline"]["achieved"] == pytest.approx((alg["gateup_bytes"] + alg["down_bytes"]) / 0.32e-3 / 1e9)
