#!/usr/bin/env python
"""Throughput of the NVFP4 W4A4 group-limited MoE layer on B200.

One step = one nvfp4moe_forward over one batch of tokens: route, quantise, group by
expert, gate/up grouped GEMM + SwiGLU + requantisation, down grouped GEMM + weighted
combine, BF16 output.  Default workload: the Beam-shape decode layer (16 tokens, hidden
5120, 256 experts of intermediate 2560 in 8 groups of 32, top-4 groups, top-8 experts,
x2.5), synthetic seeded inputs, random-init NVFP4 weights.

    python bench.py [--gpus N --steps K --warmup W] [--workload decode|prefill|skewed|sweepT]
    python bench.py --impl reference ...      # the CPU oracle on bounded samples

Multi-GPU (launched with torch.distributed.run): every rank holds a full replica of the
layer and routes its own batch (data parallel, no collective on the data path; weak
scaling); the reported time is the maximum over ranks.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import WORKLOADS, BEAM, LayerShape, activations, router_weight, expert_weight, zipf_bias  # noqa: E402

METRIC = "NVFP4 MoE-layer tokens/s; % of FP4 tensor peak (prefill) / HBM BW (decode)"
FP4_OVER_BF16 = 9.0 / 2.25          # nominal dense FP4 : BF16 tensor ratio
HBM_SPEC_GBS = 7700.0               # nominal HBM3e bandwidth of a B200 (HGX figure), a second reference
E2M1_BYTES = 0.5                    # per value
E4M3_PER16 = 1.0 / 16.0             # block-scale bytes per value


RESIDUAL_STEP = 30   # residual step k of the timed fused-residual forward (a mid-depth MoE block)


def kernel_source_hash() -> str:
    """SHA-256 over the sources of the grouped GEMM kernels (ties a stored ncu traffic figure
    to the kernel version it was measured on)."""
    import hashlib
    h = hashlib.sha256()
    for name in ("gemm.cu", "gemm.h", "common.cuh"):
        with open(os.path.join(ROOT, "nvfp4_quantized_moe_group_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemm_experts_decode_traffic.txt")


def stored_traffic(workload: str, experts_hit: int):
    """DRAM bytes per launch of the decode layer's grouped-GEMM launch (both GEMMs) from the
    committed ncu summary, scaled to this run's experts hit (traffic is proportional to the
    weight tiles streamed); None when the summary was taken on other kernel sources or another
    workload."""
    path = TRAFFIC_FILE
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if len(line) >= 2:
                vals[line[0]] = line[1]
    if vals.get("source_sha256") != kernel_source_hash() or vals.get("workload") != workload:
        return None
    return float(vals["dram_bytes_per_launch"]) / float(vals["experts_hit"]) * experts_hit


def traffic_note(workload: str) -> str:
    """Where the roofline's traffic figure comes from, or why there is none."""
    name = os.path.relpath(TRAFFIC_FILE, ROOT)
    if not os.path.exists(TRAFFIC_FILE):
        return f"no ncu summary ({name} absent)"
    vals = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if len(line) >= 2:
                vals[line[0]] = line[1]
    if vals.get("workload") != workload:
        return f"none: {name} covers the {vals.get('workload')} workload, not {workload}"
    if vals.get("source_sha256") != kernel_source_hash():
        return (f"none: {name} was captured on GEMM sources hashing to {vals.get('source_sha256', '?')[:12]}, "
                f"these hash to {kernel_source_hash()[:12]} (counters not retaken since the change)")
    return f"{name}: one ncu capture, scaled by the experts hit"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def intermediate_scales(shape: LayerShape) -> np.ndarray:
    """Static SwiGLU-intermediate global scales written by the oracle calibration script
    (the tiny layer's own file; Beam-shape layers use the Beam file's first E entries)."""
    from workloads import TINY
    name = "tiny" if shape == TINY else "beam"
    E = shape.E
    path = os.path.join(ROOT, "tests", "golden", f"intermediate_scales_{name}.txt")
    vals = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if line:
                vals.append(int(line[1], 16))
    return np.array(vals, dtype=np.uint32).view(np.float32)[:E]


# ------------------------------------------------------------------- clocks ----

_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}


_SAMPLER_CODE = r"""
import sys, time, pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[1]))
period = float(sys.argv[2])
get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    try:
        print("s", time.monotonic(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), int(get_reasons(h)),
              flush=True)
    except Exception:
        pass
    time.sleep(period)
"""


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while the timed region runs, from a
    child process (a thread here would wait on the interpreter lock while the main thread
    launches kernels)."""

    def __init__(self, device_index: int, period_s: float = 0.025):
        import subprocess
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._device = device_index
        self._proc = None
        self._lines = []
        self._thread = None
        try:
            import pynvml  # noqa: F401  (only to know that the child can use it)
            self._proc = subprocess.Popen([sys.executable, "-c", _SAMPLER_CODE, str(device_index), str(period_s)],
                                          stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            first = self._proc.stdout.readline().split()
            if first and first[0] == "max":
                self.max_mhz = int(first[1])
            else:                      # NVML could not start in the child
                self._proc.wait()
                self._proc = None
        except Exception:
            self._proc = None

    def _reader(self):
        for line in self._proc.stdout:
            self._lines.append(line)

    def __enter__(self):
        self._t0 = time.monotonic()
        if self._proc is not None:
            self._lines.clear()
            self._thread = threading.Thread(target=self._reader, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        t1 = time.monotonic()
        if self._proc is not None:
            # one more sample from this process at the end of the region (a short region can
            # fall between two of the child's samples)
            try:
                import pynvml
                pynvml.nvmlInit()
                h = pynvml.nvmlDeviceGetHandleByIndex(self._device)
                get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
                self._lines.append(f"s {t1} {pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)} "
                                   f"{int(get_reasons(h))}")
            except Exception:
                pass
            self._proc.terminate()
            self._proc.wait()
            self._thread.join()
            for line in self._lines:   # samples taken inside the region only
                f = line.split()
                if len(f) == 4 and f[0] == "s" and self._t0 <= float(f[1]) <= t1:
                    self.samples.append(int(f[2]))
                    self.reasons |= int(f[3])

    def summary(self):
        if self._proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in _REASONS.items() if self.reasons & b], "samples": len(self.samples)}


# ------------------------------------------------------------------- layer ----

def layer_shape(E: int | None) -> LayerShape:
    if E is None or E == BEAM.E:
        return BEAM
    # same hidden / intermediate sizes, fewer experts (8 groups): a smaller layer for profiling
    return LayerShape(H=BEAM.H, I=BEAM.I, E=E, n_groups=8, topk_groups=4, topk=8, routed_scale=2.5,
                      wr_std=BEAM.wr_std, w_std=BEAM.w_std)


def build_layer(moe, shape: LayerShape):
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                       shape.routed_scale)
    ex = moe.Experts(cfg)
    g_h = intermediate_scales(shape)
    for e in range(shape.E):
        ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")),
                         float(g_h[e]))
    torch.cuda.synchronize()
    return cfg, ex


def algorithmic(shape: LayerShape, T: int, counts: np.ndarray):
    """Algorithmic bytes / FLOPs of one step, from the routing the step actually produced.
    Per GEMM: its weights (codes, E4M3 scales, FP32 globals) of the experts hit plus its NVFP4
    A operand (gate/up also the requantised h it writes); the down GEMM's FP32 combine into the
    accumulator is implementation traffic and not counted."""
    H, I, k = shape.H, shape.I, shape.topk
    hit = int((counts > 0).sum())
    pairs = T * k
    per_val = E2M1_BYTES + E4M3_PER16                      # 0.5625 bytes per NVFP4 value
    w13 = 2 * I * H * per_val + 8                          # gate + up codes, scales, globals
    wd = H * I * per_val + 8
    gateup_bytes = hit * w13 + pairs * H * per_val + pairs * I * per_val
    down_bytes = hit * wd + pairs * I * per_val
    layer_bytes = hit * (w13 + wd) + T * H * 2 + T * H * 2 + shape.E * H * 4
    flops = 2.0 * pairs * (2 * I * H + H * I)
    gateup_flops = 2.0 * pairs * 2 * I * H
    down_flops = 2.0 * pairs * H * I
    return {"experts_hit": hit, "gateup_bytes": gateup_bytes, "down_bytes": down_bytes, "layer_bytes": layer_bytes,
            "flops": flops, "gateup_flops": gateup_flops, "down_flops": down_flops}


def fp4_peaks(p: dict) -> tuple[float, float]:
    """Dense FP4 tensor peak in TFLOP/s: the measured BF16 GEMM peak times the nominal
    FP4 : BF16 ratio, burst (a kernel timed alone or a step of milliseconds) and sustained (a
    seconds-long loop under the power cap)."""
    return p["bf16_tflops"] * FP4_OVER_BF16, p["bf16_tflops_sustained"] * FP4_OVER_BF16


def kernel_roofline(nbytes: float, flops: float, ms: float, p: dict) -> dict:
    """One kernel against the roofline that binds it: HBM (bytes over the measured copy
    bandwidth) or FP4 tensor (FLOPs over the burst FP4 peak), whichever takes longer; both
    fractions are given, and the FP4 one also against the sustained peak."""
    burst, sustained = fp4_peaks(p)
    s = ms / 1e3
    t_bytes = nbytes / (p["hbm_gbs"] * 1e9)
    t_flops = flops / (burst * 1e12)
    gbs = nbytes / s / 1e9
    tflops = flops / s / 1e12
    out = {"ms": ms, "bytes": nbytes, "flops": flops, "gbs": gbs, "tflops": tflops,
           "hbm_frac": gbs / p["hbm_gbs"], "fp4_frac": tflops / burst, "fp4_frac_sustained": tflops / sustained}
    if t_bytes >= t_flops:
        out.update({"bound": "hbm", "achieved": gbs, "peak": p["hbm_gbs"], "unit": "GB/s",
                    "frac_of_spec": gbs / HBM_SPEC_GBS})
    else:
        out.update({"bound": "tensor", "achieved": tflops, "peak": burst, "unit": "TFLOP/s"})
    out["frac"] = out["achieved"] / out["peak"]
    return out


def run_fp8(moe, shape: LayerShape, cfg, x, wr, bias, T: int, steps: int, warmup: int, world: int) -> dict:
    """The FP8 W8A8 variant of the layer (nvfp4moe_forward_fp8) on the same batch: its own
    experts quantised per output channel, K device-timed steps, and its HBM roofline (E4M3
    weights of the routed experts, one byte per value, plus FP32 channel scales)."""
    ex = moe.Fp8Experts(cfg)
    for e in range(shape.E):
        ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")))
    ws = torch.empty(moe.forward_fp8_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, shape.H), dtype=torch.bfloat16, device="cuda")
    _, dbg = moe.forward_fp8(ex, x, wr, bias, out=out, ws=ws, debug=True)
    st = moe.status_read(ws)
    if st != moe.OK:
        raise RuntimeError(f"fp8 forward status {moe.status_string(st)}")
    hit = int((dbg["counts"].cpu().numpy() > 0).sum())
    launches = moe.last_launch_count()
    del dbg
    for _ in range(warmup):
        moe.forward_fp8(ex, x, wr, bias, out=out, ws=ws)
    torch.cuda.synchronize()
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed_fp8")
    f0.record()
    for _ in range(steps):
        moe.forward_fp8(ex, x, wr, bias, out=out, ws=ws)
    f1.record()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier(world)
    ms = max_over_ranks(f0.elapsed_time(f1), world) / steps
    st = moe.status_read(ws)
    if st != moe.OK:
        raise RuntimeError(f"fp8 forward status {moe.status_string(st)}")
    ex.close()
    H, I = shape.H, shape.I
    w_bytes = hit * (3 * H * I + 4 * (2 * I + H))
    layer_bytes = w_bytes + T * H * 2 * 2 + shape.E * H * 4
    p = peaks()
    return {"value": tokens_per_second(world, T, steps, ms * steps), "unit": "tokens/s", "ms_per_step": ms,
            "experts_hit": hit, "gpu_launches_per_step": launches,
            "layer_roofline": {"bound": "hbm", "bytes_per_step": layer_bytes,
                               "achieved": layer_bytes / (ms / 1e3) / 1e9, "peak": p["hbm_gbs"], "unit": "GB/s",
                               "frac": layer_bytes / (ms / 1e3) / (p["hbm_gbs"] * 1e9)},
            "note": "nvfp4moe_forward_fp8: E4M3 weights with per-channel scales, per-token E4M3 activations, "
                    "tcgen05 kind::f8f6f4 grouped GEMMs; same batch and routing as the NVFP4 line"}


def e2e_pipelined(moe, ex, x_cpu, wr, bias, ws, T: int, H: int, warmup: int, steps: int, world: int) -> float:
    """Device time of ``steps`` forwards fed from pinned host memory: per step one host-to-device
    copy of the step's tokens and one device-to-host copy of its output, on a copy stream with
    two buffers each, overlapped with the neighbouring steps' compute.  Returns the elapsed
    milliseconds (max over ranks), from before the first copy in to after the last copy out."""
    stream = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    x_host = x_cpu.pin_memory()
    out_host = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    out_dev = [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    h2d = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        copy.wait_stream(stream)
        with torch.cuda.stream(copy):
            for b in range(min(2, n)):
                x_dev[b].copy_(x_host, non_blocking=True)
                h2d[b].record(copy)
        for k in range(n):
            b = k & 1
            stream.wait_event(h2d[b])
            moe.forward(ex, x_dev[b], wr, bias, out=out_dev[b], ws=ws)
            done[b].record(stream)
            copy.wait_event(done[b])
            with torch.cuda.stream(copy):
                out_host[b].copy_(out_dev[b], non_blocking=True)
                if k + 2 < n:
                    x_dev[b].copy_(x_host, non_blocking=True)
                    h2d[b].record(copy)
        stream.wait_stream(copy)

    run(warmup)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world)


def _oracle_cfg(shape: LayerShape):
    import types
    return types.SimpleNamespace(E=shape.E, n_groups=shape.n_groups, topk_groups=shape.topk_groups,
                                 topk=shape.topk, routed_scale=shape.routed_scale)


def _blas_threads() -> int:
    from threadpoolctl import threadpool_info
    return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])


def _oracle_experts(shape: LayerShape, experts):
    """NVFP4 weights of the given experts, quantised by the oracle (the oracle's counterpart of
    nvfp4moe_experts_create: prepared once, outside any timed region)."""
    import oracle
    return {e: tuple(oracle.quantize_tensor(expert_weight(shape, e, n).float().numpy())
                     for n in ("gate", "up", "down")) for e in experts}


def cpu_baseline_oracle(shape: LayerShape, wl, x_cpu, wr_cpu, bias_cpu, n_tokens=5):
    """The oracle on a bounded sample of the step: routing and input quantisation of every
    token, then the layer output of ``n_tokens`` tokens (their 8 experts' FP64 SwiGLU MLPs on
    dequantised weights).  Expert weights are quantised beforehand, untimed, as the library's
    experts are."""
    import oracle
    g_h = intermediate_scales(shape)
    cfg = _oracle_cfg(shape)
    x = x_cpu.float().numpy()
    t0 = time.perf_counter()
    r = oracle.route(x.astype(np.float64), wr_cpu.numpy(), cfg, None if bias_cpu is None else bias_cpu.numpy())
    xc, xs, gx = oracle.quantize(x)
    elapsed = time.perf_counter() - t0
    toks = list(range(min(n_tokens, wl.T)))
    qex = _oracle_experts(shape, sorted({int(e) for t in toks for e in r.idx[t]}))
    t0 = time.perf_counter()
    for t in toks:
        xhat = oracle.dequantize(xc[t:t + 1], xs[t:t + 1], gx)
        for j in range(shape.topk):
            e = int(r.idx[t, j])
            oracle.expert_mlp(xhat, *qex[e], np.float32(g_h[e]))
    elapsed += time.perf_counter() - t0
    return {"value": len(toks) / elapsed, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"routing + input quantisation of all {wl.T} tokens and the layer output of {len(toks)} "
                      f"token(s) ({shape.topk} experts each, FP64 MLP on dequantised NVFP4 weights; weight "
                      f"quantisation done beforehand, untimed); {elapsed:.1f} s of CPU work"}


# --------------------------------------------------------------------- main ----

def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def tokens_per_second(world: int, tokens_per_rank: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput: tokens of every rank over the slowest rank's time."""
    return world * tokens_per_rank * steps / (elapsed_ms / 1e3)


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


CONFIG_WORKLOADS = ("prefill", "skewed", "sweep32768")   # the compute-heavy configs beside the headline


def timed_steps(fn, steps: int, world: int, stream=None) -> float:
    """Device time of ``steps`` calls of fn (CUDA events on the launching stream, a barrier and a
    synchronize on both sides), max over ranks, in milliseconds."""
    stream = stream if stream is not None else torch.cuda.current_stream()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for k in range(steps):
        fn(k)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(start.elapsed_time(stop), world)


def measure_workload(moe, ex, shape: LayerShape, wl, x, wr, bias, steps: int, warmup: int, world: int,
                     clock=None) -> dict:
    """One workload on the layer: K device-timed forwards with nothing recorded between their
    launches (the figure the line reports), then K more with CUDA events around each
    grouped GEMM (their durations, for the kernel rooflines), then a stage breakdown from
    steps with every stage bracketed.  ``clock``: a ClockSampler to run over the first region."""
    import contextlib
    T = wl.T
    out = torch.empty((T, shape.H), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.forward_workspace_bytes(ex.cfg, T), dtype=torch.uint8, device="cuda")
    _, dbg = moe.forward(ex, x, wr, bias, out=out, ws=ws, debug=True)
    st = moe.status_read(ws)
    if st != moe.OK:
        raise RuntimeError(f"{wl.name}: forward status {moe.status_string(st)}")
    alg = algorithmic(shape, T, dbg["counts"].cpu().numpy())
    launches = moe.last_launch_count()
    del dbg
    for _ in range(warmup):
        moe.forward(ex, x, wr, bias, out=out, ws=ws)
    torch.cuda.synchronize()
    with (clock if clock is not None else contextlib.nullcontext()):
        torch.cuda.nvtx.range_push("timed")
        elapsed = timed_steps(lambda k: moe.forward(ex, x, wr, bias, out=out, ws=ws), steps, world)
        torch.cuda.nvtx.range_pop()
    # the grouped GEMMs' durations, from a second region of the same steps with events around
    # them: with short segments one launch runs both (the GATEUP events bracket it, DOWN is
    # empty), else two launches, each bracketed
    one_launch = T * shape.topk < 32 * shape.E          # the library's rule (nvfp4moe_debug.separate_gemms)
    timers = [moe.StageTimer(("gateup", "down")) for _ in range(steps)]
    ev_elapsed = timed_steps(lambda k: moe.forward(ex, x, wr, bias, out=out, ws=ws, timer=timers[k]), steps, world)
    gemm_ms = {n: max_over_ranks(statistics.mean(t.stage_ms()[n] for t in timers), world) for n in ("gateup", "down")}
    sep_elapsed = None
    if one_launch:
        experts_ms = gemm_ms["gateup"] + gemm_ms["down"]
        # for context: the same GEMMs as two launches, each timed
        timers = [moe.StageTimer(("gateup", "down")) for _ in range(steps)]
        for k in range(warmup):
            moe.forward(ex, x, wr, bias, out=out, ws=ws, separate_gemms=True)
        sep_elapsed = timed_steps(lambda k: moe.forward(ex, x, wr, bias, out=out, ws=ws, timer=timers[k],
                                                        separate_gemms=True), steps, world)
        gemm_ms = {n: max_over_ranks(statistics.mean(t.stage_ms()[n] for t in timers), world)
                   for n in ("gateup", "down")}
    full = [moe.StageTimer() for _ in range(min(steps, 20))]
    for t in full:
        moe.forward(ex, x, wr, bias, out=out, ws=ws, timer=t)
    torch.cuda.synchronize()
    stage = {n: statistics.mean(t.stage_ms()[n] for t in full) for n in moe.STAGES if n not in ("amax", "gather")}
    st = moe.status_read(ws)
    if st != moe.OK:
        raise RuntimeError(f"{wl.name}: forward status {moe.status_string(st)}")
    p = peaks()
    ms = elapsed / steps
    burst, sustained = fp4_peaks(p)
    layer_s = ms / 1e3
    res = {
        "workload": wl.describe(), "T_per_rank": T, "experts_hit": alg["experts_hit"], "ms_per_step": ms,
        "value": tokens_per_second(world, T, steps, elapsed), "unit": "tokens/s",
        "gpu_launches_per_step": launches, "alg": alg, "stage_ms": stage,
        "gemm_region_ms_per_step": ev_elapsed / steps,
        "gemms": {"gateup": kernel_roofline(alg["gateup_bytes"], alg["gateup_flops"], gemm_ms["gateup"], p),
                  "down": kernel_roofline(alg["down_bytes"], alg["down_flops"], gemm_ms["down"], p)},
    }
    if one_launch:
        res["experts_kernel"] = kernel_roofline(alg["gateup_bytes"] + alg["down_bytes"],
                                                alg["gateup_flops"] + alg["down_flops"], experts_ms, p)
        res["dominant"] = {**res["experts_kernel"], "kernel": EXPERTS_KERNEL}
        res["gemms"]["note"] = (f"the same step with the two GEMMs as two launches (nvfp4moe_debug.separate_gemms), "
                                f"each timed with CUDA events: {sep_elapsed / steps:.4f} ms per step")
    else:
        res["dominant"] = {**res["gemms"]["gateup"], "kernel": GATEUP_KERNEL}
    res.update({
        "layer_roofline": {"bytes_per_step": alg["layer_bytes"], "flops_per_step": alg["flops"],
                           "hbm_frac": alg["layer_bytes"] / layer_s / (p["hbm_gbs"] * 1e9),
                           "fp4_frac": alg["flops"] / layer_s / (burst * 1e12),
                           "fp4_frac_sustained": alg["flops"] / layer_s / (sustained * 1e12),
                           "tflops": alg["flops"] / layer_s / 1e12},
        "_ws": ws, "_out": out,
    })
    return res


EXPERTS_KERNEL = ("moe_gemm_kernel<fused, decode> (one persistent launch of both tcgen05 mxf4nvf4 grouped GEMMs: "
                  "gate/up + SwiGLU + requant, down + combine)")
GATEUP_KERNEL = "moe_gemm_kernel<gate/up> (tcgen05 mxf4nvf4 grouped GEMM + SwiGLU + requant)"


def config_entry(m: dict, wl) -> dict:
    """The JSON object of one compute-heavy config: its step time and throughput, stage times,
    the roofline of its dominant kernel (with full segments the gate/up GEMM, two thirds of the
    FLOPs and weight bytes; with short ones the launch that runs both GEMMs), both GEMMs'
    rooflines, and the whole layer against both rooflines."""
    k = m["dominant"]
    return {"workload": m["workload"], "T_per_rank": m["T_per_rank"], "experts_hit": m["experts_hit"],
            "ms_per_step": m["ms_per_step"], "value": m["value"], "unit": "tokens/s",
            "stage_ms": m["stage_ms"], "roofline": {**{n: k[n] for n in ("bound", "achieved", "peak", "unit", "frac")},
                                                    "kernel": k["kernel"], "traffic": None},
            "gemms": m["gemms"], "layer_roofline": m["layer_roofline"],
            "l2": "no flush: every step streams the routed experts' weights "
                  f"({m['alg']['layer_bytes'] / 1e9:.2f} GB > 126 MB L2)"}


def run_ours(args, world, rank, local):
    import nvfp4_quantized_moe_group_b200 as moe
    wl = WORKLOADS[args.workload]
    shape = layer_shape(args.experts) if args.experts else wl.shape
    T = wl.T
    cfg, ex = build_layer(moe, shape)
    x_cpu = activations(T, shape, seed=wl.seed + rank, rms_rows=wl.rms_rows)
    wr_cpu = router_weight(shape)
    bias_cpu = zipf_bias(shape.E) if wl.zipf else None
    x = x_cpu.cuda()
    wr = wr_cpu.cuda()
    bias = None if bias_cpu is None else bias_cpu.cuda()
    stream = torch.cuda.current_stream()

    # ---- the headline workload: device-timed steps with inputs resident in HBM and nothing
    # recorded between launches, then the GEMMs' durations and the stage breakdown
    clocks = ClockSampler(local, args.clock_period_ms / 1000.0)
    m = measure_workload(moe, ex, shape, wl, x, wr, bias, args.steps, args.warmup, world, clock=clocks)
    ws, out = m.pop("_ws"), m.pop("_out")
    alg = m["alg"]

    # ---- end to end: pinned host input -> device, forward, device -> pinned host output.  Every
    # step copies its tokens in and its output rows out; the copies run on a second stream,
    # double-buffered, so that step k+1's input and step k-1's output move while step k computes
    e2e_ms = e2e_pipelined(moe, ex, x_cpu, wr, bias, ws, T, shape.H, args.warmup, args.steps, world)

    # ---- the same step replayed from a CUDA graph (one capture, K replays; launch cost removed)
    graph = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream()
    cap_stream.wait_stream(stream)
    with torch.cuda.graph(graph, stream=cap_stream):
        moe.forward(ex, x, wr, bias, out=out, ws=ws)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    graph_ms = timed_steps(lambda k: graph.replay(), args.steps, world)
    del graph
    st = moe.status_read(ws)
    if st != moe.OK:
        raise RuntimeError(f"forward status after graph replay {moe.status_string(st)}")

    # ---- the layer fused with its residual-stream neighbours (RMSNorm in, weighted add out)
    h_res = (x.float() * 3.0).to(torch.bfloat16)
    gamma = torch.ones(shape.H, dtype=torch.float32, device="cuda")
    h_out = torch.empty_like(h_res)
    for _ in range(args.warmup):
        moe.forward_residual(ex, h_res, gamma, 1e-6, RESIDUAL_STEP, wr, bias, out=h_out, ws=ws)
    torch.cuda.synchronize()
    residual_ms = timed_steps(lambda k: moe.forward_residual(ex, h_res, gamma, 1e-6, RESIDUAL_STEP, wr, bias,
                                                             out=h_out, ws=ws), args.steps, world)
    st = moe.status_read(ws)
    if st != moe.OK:
        raise RuntimeError(f"residual forward status {moe.status_string(st)}")
    del ws, out

    fp8 = None if args.no_fp8 else run_fp8(moe, shape, cfg, x, wr, bias, T, args.steps, args.warmup, world)

    # ---- the compute-heavy configs on the same layer (prefill, skewed routing, the largest
    # token count of the sweep) and the standalone activation quantisation
    configs = {}
    if not args.no_configs and not args.experts and wl.shape == BEAM:
        # the standalone quantisation first: issue-bound, it is measured before the long
        # GEMM-bound configs have brought the power cap in
        qclk = ClockSampler(local, args.clock_period_ms / 1000.0)
        q = measure_quantize(moe, args.steps, args.warmup, world, rank, clock=qclk)
        quant_entry = {**{k: q[k] for k in ("workload", "ms_per_step", "value", "unit", "roofline")},
                       "clocks": qclk.summary()}
        for name in CONFIG_WORKLOADS:
            cw = WORKLOADS[name]
            xc = activations(cw.T, shape, seed=cw.seed + rank, device="cuda")
            bc = zipf_bias(shape.E).cuda() if cw.zipf else None
            cclk = ClockSampler(local, args.clock_period_ms / 1000.0)
            cm = measure_workload(moe, ex, shape, cw, xc, wr, bc, args.steps, args.warmup, world, clock=cclk)
            cm.pop("_ws"), cm.pop("_out")
            configs[name] = {**config_entry(cm, cw), "clocks": cclk.summary()}
            del xc
            torch.cuda.empty_cache()
        configs["quantize"] = quant_entry

    p = peaks()
    gu = m["dominant"]
    roof = {k: gu[k] for k in ("bound", "achieved", "peak", "unit", "frac")}
    if roof["bound"] == "hbm":
        roof["frac_of_spec"] = gu["frac_of_spec"]
        roof["spec_peak"] = HBM_SPEC_GBS
    roof["traffic"] = stored_traffic(args.workload if not args.experts else f"{args.workload}-e{shape.E}",
                                     alg["experts_hit"])
    roof["traffic_source"] = traffic_note(args.workload if not args.experts else f"{args.workload}-e{shape.E}")
    roof["kernel"] = gu["kernel"]
    roof["duration_source"] = (f"CUDA events around the GEMM launch of each of {args.steps} steps of a second "
                               "timed region right after the headline one (same inputs), on the launching stream")
    roof["peak_source"] = (f"{p['source']} hbm_gbs (a copy bandwidth: a read-only stream can exceed it slightly)"
                           if roof["bound"] == "hbm"
                           else f"{p['source']} bf16_tflops (burst) x {FP4_OVER_BF16:g} (nominal FP4:BF16)")
    res = {
        "metric": METRIC, "value": m["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, fp32 accumulate)",
        "data": "synthetic (seeded counter-hash inputs; random-init NVFP4 weights)",
        "config": {"workload": wl.describe() if not args.experts else wl.describe() + f" (E={shape.E} variant)",
                   "T_per_rank": T, "experts_hit": alg["experts_hit"], "parallelism": f"dp{world} (replicas)",
                   "l2": "no flush: every step streams the routed experts' weights "
                         f"({alg['layer_bytes'] / 1e9:.2f} GB > 126 MB L2)"},
        "roofline": roof, "layer_roofline": {**m["layer_roofline"],
                                             "hbm_frac_of_spec": m["layer_roofline"]["hbm_frac"] * peaks()["hbm_gbs"]
                                             / HBM_SPEC_GBS},
        "gemms": m["gemms"],
        **({"experts_kernel": m["experts_kernel"]} if "experts_kernel" in m else {}),
        "stage_ms": m["stage_ms"],
        "e2e": {"value": tokens_per_second(world, T, args.steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * shape.H * 2, "d2h_bytes_per_step": T * shape.H * 2},
        "gpu_launches": m["gpu_launches_per_step"] * args.steps,
        "clocks": clocks.summary(),
        "residual": {"value": tokens_per_second(world, T, args.steps, residual_ms), "unit": "tokens/s",
                     "ms_per_step": residual_ms / args.steps, "step_k": RESIDUAL_STEP,
                     "note": "nvfp4moe_forward_residual: RMSNorm of the residual stream, the layer, and "
                             "the weighted residual add in finalize"},
        "graph": {"value": tokens_per_second(world, T, args.steps, graph_ms), "unit": "tokens/s",
                  "ms_per_step": graph_ms / args.steps,
                  "note": "the same forward captured once in a CUDA graph and replayed K times"},
    }
    if configs:
        res["configs"] = configs
    if fp8 is not None:
        res["fp8"] = fp8
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_oracle(shape, wl, x_cpu, wr_cpu, bias_cpu)
    ex.close()
    return res


QUANT_ROWS = 32768


def measure_quantize(moe, steps: int, warmup: int, world: int, rank: int, clock=None) -> dict:
    """Standalone quantize_nvfp4 on 32768 x 5120 BF16 activations with a dynamic global scale
    and swizzled scales: the amax pass reads x once, the quantise pass reads it again and
    writes codes + scales, so the algorithmic bytes are 2 * 2 * rows * cols + rows * cols * 9/16."""
    import contextlib
    rows, cols = QUANT_ROWS, BEAM.H
    x = activations(rows, BEAM, seed=rank, device="cuda")
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(moe.swizzled_scale_bytes(rows, cols // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.quantize_workspace_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    for _ in range(warmup):
        moe.quantize(x, swizzled=True, ws=ws, out=(codes, scales, g))
    torch.cuda.synchronize()
    with (clock if clock is not None else contextlib.nullcontext()):
        elapsed = timed_steps(lambda k: moe.quantize(x, swizzled=True, ws=ws, out=(codes, scales, g)), steps, world)
    ms = elapsed / steps
    launches = moe.last_launch_count()
    if moe.status_read(ws) != moe.OK:
        raise RuntimeError("quantize status")
    nbytes = 2 * rows * cols * 2 + rows * cols // 2 + rows * cols // 16
    p = peaks()
    gbs = world * nbytes / (ms / 1e3) / 1e9
    return {"workload": f"quantize {rows}x{cols} (dynamic global scale, swizzled scales)", "ms_per_step": ms,
            "value": gbs, "unit": "GB/s", "bytes_per_step": nbytes, "launches": launches,
            "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": p["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / world / p["hbm_gbs"], "traffic": None}}


def run_quantize(args, world, rank, local):
    """The standalone quantisation as its own bench line (``--workload quantize``)."""
    import nvfp4_quantized_moe_group_b200 as moe
    clocks = ClockSampler(local, args.clock_period_ms / 1000.0)
    q = measure_quantize(moe, args.steps, args.warmup, world, rank, clock=clocks)
    return {"metric": "quantize_nvfp4 HBM GB/s (32768x5120 BF16, dynamic global scale, swizzled scales)",
            "value": q["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": q["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16->e2m1", "data": "synthetic",
            "config": {"workload": "quantize 32768x5120", "bytes_per_step": q["bytes_per_step"],
                       "l2": "input 335 MB > 126 MB L2 (no flush)"},
            "roofline": q["roofline"], "gpu_launches": q["launches"] * args.steps, "clocks": clocks.summary()}


def run_ep(args, world, rank, local):
    """The layer under expert parallelism (nvfp4_quantized_moe_group_b200.ep): rank r holds
    experts [r E/G, (r+1) E/G); a step all-gathers the ranks' tokens (NCCL), runs the rank's
    partial layer on all of them, reduce-scatters the FP32 sums (NCCL) and rounds to BF16.
    Per-rank batch: the workload's T tokens.  Roofline: this rank's share of the weight bytes
    of the experts hit by all gathered tokens, over the step time."""
    import nvfp4_quantized_moe_group_b200 as moe
    from nvfp4_quantized_moe_group_b200.ep import ExpertParallelLayer
    wl = WORKLOADS[args.workload]
    shape = layer_shape(args.experts) if args.experts else wl.shape
    T = wl.T
    cfg = moe.make_cfg(shape.E, shape.n_groups, shape.topk_groups, shape.topk, shape.H, shape.I,
                       shape.routed_scale)
    layer = ExpertParallelLayer(cfg, exchange=args.exchange)
    ex = layer.create_experts()
    g_h = intermediate_scales(shape)
    for e in range(layer.e_begin, layer.e_begin + layer.e_count):
        ex.set_from_bf16(e, *(expert_weight(shape, e, w, device="cuda") for w in ("gate", "up", "down")),
                         float(g_h[e]))
    x_cpu = activations(T, shape, seed=wl.seed + rank, rms_rows=wl.rms_rows)
    x = x_cpu.cuda()
    wr = router_weight(shape).cuda()
    bias = zipf_bias(shape.E).cuda() if wl.zipf else None
    # routing of the gathered batch: which of this rank's experts the step streams
    x_all = layer.gather(x)
    _, dbg = moe.forward_partial(ex, x_all, wr, bias, debug=True)
    counts = dbg["counts"].cpu().numpy()[layer.e_begin:layer.e_begin + layer.e_count]
    hit_local = int((counts > 0).sum())
    launches = moe.last_launch_count() + 1          # + finalize
    del dbg
    if args.exchange == "all_to_all":
        # one step with every library call's launch count added up
        counted = []

        def counting(fn):
            def call(*a, **kw):
                r = fn(*a, **kw)
                counted.append(moe.last_launch_count())
                return r
            return call

        ops = dict(layer._a2a)
        layer._a2a = {k: counting(v) for k, v in ops.items()}
        layer.forward(x, wr, bias)
        layer._a2a = ops
        launches = sum(counted)

    for _ in range(args.warmup):
        layer.forward(x, wr, bias)
    torch.cuda.synchronize()
    barrier(world)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, args.clock_period_ms / 1000.0) as clocks:
        start.record()
        for _ in range(args.steps):
            layer.forward(x, wr, bias)
        stop.record()
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(stop), world) / args.steps
    # end to end: pinned host tokens in, BF16 rows out
    x_host = x_cpu.pin_memory()
    out_host = torch.empty((T, shape.H), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        x_dev.copy_(x_host, non_blocking=True)
        out_host.copy_(layer.forward(x_dev, wr, bias), non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    p = peaks()
    per_expert = 3 * shape.H * shape.I * (E2M1_BYTES + E4M3_PER16) + 16
    local_bytes = hit_local * per_expert + world * T * shape.H * 2 + shape.E * shape.H * 4
    layer.close()
    return {"metric": METRIC, "value": tokens_per_second(world, T, 1, ms), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, fp32 accumulate)",
            "data": "synthetic (seeded counter-hash inputs; random-init NVFP4 weights)",
            "config": {"workload": wl.describe() + f" per rank, expert parallel over {world} rank(s)",
                       "T_per_rank": T, "experts_per_rank": layer.e_count, "local_experts_hit": hit_local,
                       "parallelism": f"ep{world} " + {
                           "gather": "(all-gather tokens, reduce-scatter FP32 sums)",
                           "peer": "(all-gather tokens, down GEMM adds the FP32 sums into the owning ranks' memory)",
                           "all_to_all": "(all-to-all of quantised pair rows and weighted output rows)"}[args.exchange],
                       "l2": "no flush: every step streams the rank's routed experts' weights"},
            "roofline": {"bound": "hbm", "achieved": local_bytes / (ms / 1e3) / 1e9, "peak": p["hbm_gbs"],
                         "unit": "GB/s", "frac": local_bytes / (ms / 1e3) / (p["hbm_gbs"] * 1e9), "traffic": None,
                         "note": "whole step of this rank (partial layer + collectives) on its algorithmic bytes"},
            "e2e": {"value": tokens_per_second(world, T, 1, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * shape.H * 2, "d2h_bytes_per_step": T * shape.H * 2},
            "gpu_launches": launches * args.steps, "clocks": clocks.summary()}


def run_route(args, world, rank, local):
    """Standalone route(hidden, W_router) (nvfp4moe_route) on Beam's router for T=4096 tokens:
    for T > 64 the logits run as exact int8 digit-plane products on the tensor cores (13 digit
    pairs), so the dominant kernel is bound by int8 tensor throughput; peak = measured BF16
    burst x 2 (nominal INT8 : BF16 dense ratio)."""
    import nvfp4_quantized_moe_group_b200 as moe
    T = 4096
    cfg = moe.cfg_default()
    x = activations(T, BEAM, seed=rank, device="cuda")
    wr = router_weight(BEAM).cuda()
    ws = torch.empty(moe.route_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        moe.route(cfg, x, wr, ws=ws)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    with ClockSampler(local, args.clock_period_ms / 1000.0) as clocks:
        start.record()
        for _ in range(args.steps):
            moe.route(cfg, x, wr, ws=ws)
        stop.record()
        torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), world) / args.steps
    launches = moe.last_launch_count()
    if moe.status_read(ws) != moe.OK:
        raise RuntimeError("route status")
    ops = 13 * 2.0 * T * BEAM.H * BEAM.E          # int8 digit-pair products, the dominant kernel
    p = peaks()
    i8_peak = p["bf16_tflops"] * 2
    return {"metric": "route tokens/s (Beam router, T=4096)", "value": world * T / (ms / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 x fp32 -> exact int8 digits",
            "data": "synthetic", "config": {"workload": "route T=4096, E=256, H=5120",
                                            "l2": "token digit planes 84 MB < 126 MB L2 (not flushed)"},
            "roofline": {"bound": "tensor", "achieved": ops / (ms / 1e3) / 1e12, "peak": i8_peak, "unit": "TOP/s",
                         "frac": ops / (ms / 1e3) / 1e12 / i8_peak, "traffic": None,
                         "note": "whole call (slicing, logits, top-k) against the int8 work of the logits kernel"},
            "gpu_launches": launches * args.steps, "clocks": clocks.summary()}


FP32_LANES_PER_SM = 128   # FP32 FMA lanes per B200 SM (4 partitions x 32)


def run_quantize_lh(args, world, rank, local):
    """Local-Hessian weight quantisation of one Beam expert per step: gate [2560, 5120], up
    [2560, 5120] and down [5120, 2560], m = 4 (9 candidate scales per block), local Hessian
    blocks of 256 synthetic calibration tokens.  FP32-ALU bound: per block and candidate the
    kernel does a 16x16 matrix-vector product and a dot product (272 FMAs) plus ~40 other
    operations; the roofline counts 2 x 272 FLOP per block-candidate against the FP32 FMA peak
    of the SMs at the maximum SM clock."""
    import nvfp4_quantized_moe_group_b200 as moe
    H, I, m = BEAM.H, BEAM.I, 4
    shapes = [(I, H), (I, H), (H, I)]
    mats, hess = [], []
    for j, (rows, cols) in enumerate(shapes):
        mats.append(expert_weight(BEAM, j, ("gate", "up", "down")[j], device="cuda"))
        x = activations(256, LayerShape(H=cols, I=I, E=1, n_groups=1, topk_groups=1, topk=1, routed_scale=1.0,
                                        wr_std=1.0, w_std=0.02), seed=70 + j + rank)
        # the caller's calibration statistics: the 16x16 diagonal blocks of X^T X (FP64, then FP32)
        xb = x.double().reshape(x.shape[0], cols // 16, 16)
        hess.append(torch.einsum("nbi,nbj->bij", xb, xb).float().contiguous().cuda())
    ws = torch.empty(moe.quantize_workspace_bytes(H, H), dtype=torch.uint8, device="cuda")

    def step():
        for w, hb in zip(mats, hess):
            moe.quantize_weights_lh(w, hb, m, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    with ClockSampler(local, args.clock_period_ms / 1000.0) as clocks:
        start.record()
        for _ in range(args.steps):
            step()
        stop.record()
        torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), world) / args.steps
    if moe.status_read(ws) != moe.OK:
        raise RuntimeError("local-Hessian quantize status")
    blocks = sum(r * c // 16 for r, c in shapes)
    flops = blocks * (2 * m + 1) * 2 * 272
    clk = clocks.summary()
    max_mhz = clk["sm_max_mhz"] or 1965
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    peak = sms * FP32_LANES_PER_SM * 2 * max_mhz * 1e6 / 1e12
    achieved = flops / (ms / 1e3) / 1e12
    return {"metric": "local-Hessian NVFP4 weight quantisation, Beam experts/s (m = 4)",
            "value": world * 1e3 / ms, "unit": "experts/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16->e2m1 (fp32 search)", "data": "synthetic",
            "config": {"workload": "quantize_lh: gate/up 2560x5120 + down 5120x2560, m=4, 256 calibration tokens",
                       "blocks_per_step": blocks},
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": "SMs x 128 FP32 lanes x 2 FLOP x max SM clock"},
            "gpu_launches": 2 * len(shapes) * args.steps, "clocks": clk}


def run_reference(args, world, rank):
    """The oracle as the reference arm.  Each step is a bounded sample of the workload's step:
    routing and input quantisation of all its tokens plus one (token, slot) pair's expert
    (FP64 SwiGLU MLP on dequantised NVFP4 weights); the steps cycle through the 8 pairs of
    token 0, whose experts are quantised once beforehand (untimed).  A pair is 1/topk token."""
    import oracle
    wl = WORKLOADS[args.workload]
    shape = layer_shape(args.experts) if args.experts else wl.shape
    T = wl.T
    g_h = intermediate_scales(shape)
    x = activations(T, shape, seed=wl.seed, rms_rows=wl.rms_rows).float().numpy()
    wr = router_weight(shape).numpy()
    bias = zipf_bias(shape.E).numpy() if wl.zipf else None
    cfg = _oracle_cfg(shape)
    r0 = oracle.route(x.astype(np.float64), wr, cfg, bias)
    qex = _oracle_experts(shape, [int(e) for e in r0.idx[0]])

    def step(i):
        j = i % shape.topk
        t0 = time.perf_counter()
        r = oracle.route(x.astype(np.float64), wr, cfg, bias)
        xc, xs, gx = oracle.quantize(x)
        e = int(r.idx[0, j])
        oracle.expert_mlp(oracle.dequantize(xc[:1], xs[:1], gx), *qex[e], np.float32(g_h[e]))
        return time.perf_counter() - t0

    for i in range(args.warmup):
        step(i)
    total = sum(step(args.warmup + i) for i in range(args.steps))
    value = (args.steps / shape.topk) / total
    sample = (f"each step: routing + input quantisation of all {T} tokens of the {wl.name} workload and one "
              f"(token, slot) pair's expert MLP (a pair is 1/{shape.topk} token); experts quantised beforehand")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.describe(), "T_per_rank": T},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--clock-period-ms", type=float, default=25.0,
                    help="NVML clock sampling period during the timed region")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS) + ["quantize", "quantize_lh", "route"])
    ap.add_argument("--experts", type=int, default=None, help="smaller layer with this many experts (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 W8A8 variant's measurement")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the compute-heavy configs (prefill, skewed, 32768 tokens, quantise) of the line")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the ranks (each holds E/N experts) instead of one full replica "
                         "per GPU")
    ap.add_argument("--exchange", choices=["gather", "peer", "all_to_all"], default="gather",
                    help="with --ep: all-gather the tokens and reduce-scatter FP32 sums; the same gather with the "
                         "down GEMM adding the sums into the owning ranks' memory (peer); or send each pair's "
                         "quantised row to its expert's rank and its output row back (NCCL all-to-all)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return

    world, rank, local = init_dist()
    try:
        if args.workload == "quantize":
            res = run_quantize(args, world, rank, local)
        elif args.workload == "quantize_lh":
            res = run_quantize_lh(args, world, rank, local)
        elif args.workload == "route":
            res = run_route(args, world, rank, local)
        elif args.ep:
            res = run_ep(args, world, rank, local)
        else:
            res = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
