"""Benchmark of the int4 mixture-of-experts FFN layer (libmoe_int4) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload scout_decode|scout_prefill|skewed|maverick_fp8|tiny|quantize]

One step = one full layer forward (routing, bucketing, routed SwiGLU experts,
shared expert, weighted combine) over one batch of synthetic tokens already
resident in HBM.  For N > 1 (launched by torch.distributed.run) every rank
runs an independent replica of the workload (the layer does not shard), and
the reported throughput is all ranks' tokens over the slowest rank's time.

``--workload quantize`` instead times int4_row_quantize of a 16-expert
Scout-shaped weight set (gate and up [8192, 5120], down [5120, 8192] per
expert, fp32), one step = all three projections, reported in GB/s moved.

``--impl reference`` times the CPU oracle (the plain numpy restatement of the
layer) on rank 0 on a bounded sample of the same workload; other ranks exit.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE layer tokens/s; % of HBM roofline (decode) / BF16-FP8 TC peak (prefill)"
FALLBACK_HBM_GBS = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


FALLBACK_BF16_TFLOPS = 1400.0   # sustained under the power cap


def peaks():
    """(HBM GB/s, sustained dense bf16 TFLOP/s, source)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


KERNEL_SOURCES = {   # the files a kernel's code comes from (a change invalidates its ncu numbers)
    "decode_gate_up": ["ffn_decode.cu", "ffn_decode.cuh", "common.cuh"],
    "decode_down": ["ffn_decode.cu", "ffn_decode.cuh", "common.cuh"],
    "tc_gate_up": ["tc_gemm.cu", "tc_gemm.cuh", "tcgen05.cuh", "common.cuh"],
    "tc_down": ["tc_gemm.cu", "tc_gemm.cuh", "tcgen05.cuh", "common.cuh"],
    "tc_shared_gate_up": ["tc_gemm.cu", "tc_gemm.cuh", "tcgen05.cuh", "common.cuh"],
    "tc_shared_down": ["tc_gemm.cu", "tc_gemm.cuh", "tcgen05.cuh", "common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "int4_quantized_expert_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the
    committed ncu summary, or None if absent or taken on another source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p) or kernel not in KERNEL_SOURCES:
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e["dram_bytes"]


QUANT_E, QUANT_D, QUANT_F = 16, 5120, 8192
QUANT_METRIC = "int4_row_quantize GB/s moved (fp32 weights read, int4 codes and fp32 scales written); % of HBM roofline"


def quant_matrices(E: int = QUANT_E):
    """(name, rows, cols) of the quantize workload: each projection of all
    E (16) experts as one [E * N, K] matrix."""
    D, F = QUANT_D, QUANT_F
    return [("gate", E * F, D), ("up", E * F, D), ("down", E * D, F)]


def quant_bytes(rows: int, cols: int, group: int = 128) -> int:
    """Algorithmic bytes of int4_row_quantize: fp32 in, codes + scales out."""
    return rows * cols * 4 + rows * cols // 2 + rows * (cols // group) * 4


def max_over_ranks(values, dev, world: int):
    """Element-wise max of per-rank floats (all ranks call it, in the same order)."""
    if world <= 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weights_text(s: synth.LayerShape, group: int = 128) -> str:
    if s.fmt == "int4":
        return "routed int4 g%d (fp32 scales, zero point 0); router and shared bf16" % group
    return "routed e4m3 rows (fp32 row scales), e4m3 per-row activations; router and shared bf16"


def workload_text(s: synth.LayerShape, group: int = 128) -> str:
    w = ("int4 g%d" % group) if s.fmt == "int4" else "fp8 e4m3 rows"
    gate = "sigmoid" if s.k == 1 else "softmax over top-%d" % s.k
    return ("%s: T=%d tokens, d_model=%d, expert d_ff=%d, E=%d routed experts (%s), top-%d %s gate, "
            "bf16 shared expert d_ff=%d%s" % (s.name, s.T, s.D, s.F, s.E, w, s.k, gate, s.F_shared,
                                               ", Zipf router bias" if s.skewed else ""))


# ---------------------------------------------------------------------------
# clocks sampled while the timed loop runs
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled every ~20 ms by
    NVML in a thread (nvidia-smi every 50 ms if NVML is unavailable), so
    that even a timed region of a fraction of a second gets samples."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index: int):
        self.proc = None
        self.samples = []          # (time, sm_mhz, max_mhz, reasons)
        self.stop_flag = threading.Event()
        self.t = None
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.reasons_fn = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
                               or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.t = threading.Thread(target=self._poll_nvml, daemon=True)
            self.t.start()
            return
        except Exception as e:  # no NVML: fall back to nvidia-smi
            log("NVML clock sampling unavailable (%s); using nvidia-smi" % e)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--id=" + uuid, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read_smi, daemon=True)
            self.t.start()
        except Exception as e:
            log("clock sampling unavailable:", e)
            self.proc = None

    def _poll_nvml(self):
        nv = self.nvml
        while not self.stop_flag.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = int(self.reasons_fn(self.h))
                reasons = {n for n, b in self.REASON_BITS.items() if bits & b}
                self.samples.append((time.time(), sm, self.max_mhz, reasons))
            except Exception:
                pass
            time.sleep(0.02)

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except (ValueError, IndexError):
                continue
            reasons = {n for n, v in zip(names, parts[4:8]) if v.lower() == "active"}
            self.samples.append((time.time(), sm, mx, reasons))

    def stop(self):
        self.stop_flag.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:
            # a timed region shorter than the sampling period: the samples
            # taken within one period of it
            inside = [s for s in self.samples if t0 - 0.03 <= s[0] <= t1 + 0.03]
        if not inside:
            return None
        reasons = set()
        for s in inside:
            reasons |= s[3]
        return {"sm_mhz": float(np.median([s[1] for s in inside])), "sm_max_mhz": inside[-1][2],
                "reasons": sorted(reasons), "samples": len(inside)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def build_layer(shape: synth.LayerShape, seed: int, dev: torch.device, group: int = 128, rms: bool = False):
    import int4_quantized_expert_b200 as moe
    E, k, D, F, Fs = shape.E, shape.k, shape.D, shape.F, shape.F_shared
    wr = synth.router_weight(seed, E, D).to(dev)
    bias = synth.router_bias(shape)
    bias = None if bias is None else torch.from_numpy(bias).to(dev)
    sg, su, sd = (t.to(dev) for t in synth.shared_weights(seed, D, Fs))
    if shape.fmt == "int4":
        alloc = lambda n, kk: (torch.empty(E, n, kk // 2, dtype=torch.uint8, device=dev),
                               torch.empty(E, n, kk // group, dtype=torch.float32, device=dev))
        quant = lambda w, out: moe.quantize_int4(w, group_size=group, out=out)
        fmt = moe.FMT_INT4
    else:
        alloc = lambda n, kk: (torch.empty(E, n, kk, dtype=torch.uint8, device=dev),
                               torch.empty(E, n, dtype=torch.float32, device=dev))
        quant = lambda w, out: moe.quantize_fp8_rows(w, out=out)
        fmt = moe.FMT_FP8
    gamma = synth.rms_weight(seed, D).to(dev) if rms else None
    gate, up, down = alloc(F, D), alloc(F, D), alloc(D, F)
    # Routed experts: N(0, 0.02) fp32 drawn on the device by torch's seeded
    # Philox generator (the same distribution as the parity tests' PCG64
    # draws, without minutes of host work for 128 experts), then quantized by
    # the library.  Routing depends only on x and the router, drawn as in the
    # tests.
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    wbuf = torch.empty(max(F * D, D * F), dtype=torch.float32, device=dev)
    for e in range(E):
        for (n, kk), (c, s) in (((F, D), gate), ((F, D), up), ((D, F), down)):
            w = wbuf[:n * kk].view(n, kk)
            torch.randn(n, kk, generator=gen, out=w).mul_(synth.WEIGHT_STD)
            quant(w, (c[e], s[e]))
    del wbuf
    torch.cuda.synchronize()
    layer = moe.MoELayer(E=E, k=k, D=D, F=F, F_shared=Fs, w_router=wr, router_bias=bias, gate=gate,
                         up=up, down=down, shared=(sg, su, sd), fmt=fmt, T_max=shape.T, group_size=group,
                         rms_weight=gamma, rms_eps=1e-5)
    x = synth.tokens(seed, shape.T, D).to(dev)
    return layer, x, (wr, bias, gamma)


def kernel_work(shape: synth.LayerShape, n_touched: int, group: int = 128) -> dict:
    """Algorithmic work per launch of each kernel, as (kind, amount):
    ("bytes", HBM bytes with every weight byte of a touched expert and of the
    shared expert read once and every activation read and written once) for
    the weight-streaming kernels, ("flops", 2 * multiply-adds) for the
    tensor-core ones."""
    T, D, F, Fs, E, k = shape.T, shape.D, shape.F, shape.F_shared, shape.E, shape.k
    S = T * k
    codes_gu = 2 * F * D // 2
    scales_gu = 2 * F * (D // group) * 4
    codes_d = D * F // 2
    scales_d = D * (F // group) * 4
    if shape.fmt == "fp8":   # e4m3 routed experts: one tensor-core pass each, bf16-equivalent flop count
        return {
            "rmsnorm": ("bytes", T * D * 2 * 2 + D * 2),
            "router": ("flops", 2 * T * D * E),
            "bucket": ("bytes", S * 4 * 3 + (E + 1) * 8),
            "bucket_scan": ("bytes", (E + 1) * 8),
            "bucket_place": ("bytes", S * 4 * 3),
            "quantize_x": ("bytes", T * D * 2 + S * D),
            "tc_gate_up": ("flops", 2 * S * D * 2 * F),
            "quantize_h": ("bytes", S * F * 2 * 2 + S * F),
            "tc_down": ("flops", 2 * S * F * D),
            "tc_shared_gate_up": ("flops", 2 * T * D * 2 * Fs),
            "tc_shared_down": ("flops", 2 * T * Fs * D),
            "combine": ("bytes", (S + T) * D * 4 + T * D * 2),
        }
    return {
        "rmsnorm": ("bytes", T * D * 2 * 2 + D * 2),
        "router": ("flops", 2 * T * D * E),
        "bucket": ("bytes", S * 4 * 3 + (E + 1) * 8),
        "bucket_scan": ("bytes", (E + 1) * 8),
        "bucket_place": ("bytes", S * 4 * 3),
        "act16_x": ("bytes", T * D * 2 * 2),
        # weights once; x read; h written as bf16 (routed and shared) and as the
        # down pass's fp16 operands (routed)
        "decode_gate_up": ("bytes", n_touched * (codes_gu + scales_gu) + 2 * Fs * D * 2 + T * D * 2
                           + (S * F + T * Fs) * 2 + S * F * 2),
        # weights once; h read; y written (routed and shared); out written
        "decode_down": ("bytes", n_touched * (codes_d + scales_d) + D * Fs * 2 + (S * F + T * Fs) * 2
                        + (S + T) * D * 4 + T * D * 2),
        "gather": ("bytes", S * D * 2 * 2),
        "tc_gate_up": ("flops", 2 * S * D * 2 * F),
        "tc_down": ("flops", 2 * S * F * D),
        "tc_shared_gate_up": ("flops", 2 * T * D * 2 * Fs),
        "tc_shared_down": ("flops", 2 * T * Fs * D),
    }


def layer_flops(shape: synth.LayerShape) -> int:
    T, D, F, Fs, E, k = shape.T, shape.D, shape.F, shape.F_shared, shape.E, shape.k
    return 2 * T * D * E + 2 * T * k * 3 * D * F + 2 * T * 3 * D * Fs


def run_ours(args, rank: int, world: int, dev: torch.device):
    import int4_quantized_expert_b200 as moe
    shape = synth.SHAPES[args.workload]
    layer, x, (wr, bias, gamma) = build_layer(shape, args.seed + 0, dev, args.group_size, args.rmsnorm)
    # the experts the layer's routing touches (it routes RMSNorm(x) when the layer has the norm)
    r = moe.route(x if gamma is None else moe.rmsnorm(x, gamma, 1e-5), wr, bias, shape.k)
    n_touched = int((r["counts"] > 0).sum().item())
    names = layer.launch_names(shape.T)
    out = torch.empty(shape.T, shape.D, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)    # > 126 MB L2
    stream = torch.cuda.current_stream()

    def new_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        for e in evs:
            e.record(stream)          # create the underlying cudaEvent_t
        return evs

    for _ in range(args.warmup):
        flush.zero_()
        layer.forward(x, out)
    torch.cuda.synchronize()
    assert layer.device_status() == moe.Status.OK

    # timed steps: one event pair around each layer forward (events between
    # the layer's launches would serialise kernels that otherwise overlap)
    steps_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for e0, e1 in steps_ev:
        flush.zero_()                 # L2 flushed between steps (outside the step's events)
        e0.record(stream)
        layer.forward(x, out)
        e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.summary(t_wall0, t_wall1) if sampler else None
    if sampler:
        sampler.stop()
    status = layer.device_status()
    if status != moe.Status.OK:
        raise RuntimeError("device status %d after the timed loop" % status)
    step_ms = np.array([a.elapsed_time(b) for a, b in steps_ev])
    ms = max_over_ranks([float(step_ms.mean())], dev, world)[0]

    # per-kernel times: a separate pass with an event before every launch
    n_pk = max(3, min(args.steps, 200))
    events = [new_events() for _ in range(n_pk)]
    for i in range(n_pk):
        flush.zero_()
        layer.forward_timed(x, out, events[i])
    torch.cuda.synchronize()
    per_kernel = np.zeros(len(names))
    for evs in events:
        for j in range(len(names)):
            per_kernel[j] += evs[j].elapsed_time(evs[j + 1])
    per_kernel /= n_pk

    # end to end through the host-buffer entry point (copies inside the timed region)
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    n_e2e = max(3, min(args.steps, 200))
    for _ in range(3):
        layer.forward_host(xh, oh)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for _ in range(n_e2e):
        flush.zero_()
        e0.record(stream)
        layer.forward_host(xh, oh)
        e1.record(stream)
        e1.synchronize()
        e2e_ms += e0.elapsed_time(e1)
    e2e_ms = max_over_ranks([e2e_ms / n_e2e], dev, world)[0]

    work = kernel_work(shape, n_touched, args.group_size)
    dom = int(np.argmax(per_kernel))
    dom_name = names[dom]
    hbm_peak, tc_peak, peak_src = peaks()
    kind, amount = work[dom_name]
    if kind == "bytes":
        roof = {"bound": "hbm", "kernel": dom_name, "achieved": amount / (per_kernel[dom] * 1e-3) / 1e9,
                "peak": hbm_peak, "peak_source": peak_src + " copy bandwidth", "unit": "GB/s",
                "traffic": None, "algorithmic_bytes": amount}
    else:
        fp8_kernel = shape.fmt == "fp8" and dom_name in ("tc_gate_up", "tc_down")
        peak = tc_peak * (2.0 if fp8_kernel else 1.0)   # e4m3: nominal 2x the bf16 rate
        roof = {"bound": "tensor", "kernel": dom_name, "achieved": amount / (per_kernel[dom] * 1e-3) / 1e12,
                "peak": peak, "unit": "TFLOP/s", "traffic": None, "algorithmic_flops": amount,
                "peak_source": peak_src + (" sustained dense bf16 x 2 (e4m3)" if fp8_kernel
                                           else " sustained dense bf16")}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic(dom_name, shape.name)
    layer_bytes = sum(a for kd, a in (work[n] for n in names) if kd == "bytes")

    result = {
        "metric": METRIC,
        "value": world * shape.T / (ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if shape.fmt == "int4" else "e4m3 (routed experts), bf16 (shared expert)",
        "data": ("synthetic (seeded; no dataset, random-init weights of the stated shapes: x, router and "
                 "shared expert from PCG64, routed experts N(0, 0.02) from torch's device generator)"),
        "config": {
            "workload": workload_text(shape, args.group_size) + (
                ", RMSNorm (eps 1e-5) of x in front" if args.rmsnorm else ""),
            "weights": weights_text(shape, args.group_size),
            "parallelism": "replicas" if world > 1 else "single GPU",
            "experts_touched": n_touched,
            "l2": "flushed between steps (256 MB write)",
        },
        "roofline": roof,
        "layer": {
            "streamed_bytes": layer_bytes,
            "flops": layer_flops(shape),
            "tflops": layer_flops(shape) / (ms * 1e-3) / 1e12,
            "per_kernel_ms": {n: float(v) for n, v in zip(names, per_kernel)},
            "per_kernel_note": "separate pass with an event before every launch (no overlap between launches)",
        },
        "e2e": {
            "value": world * shape.T / (e2e_ms * 1e-3),
            "unit": "tokens/s",
            "h2d_bytes_per_step": shape.T * shape.D * 2,
            "d2h_bytes_per_step": shape.T * shape.D * 2,
            "ms_per_step": e2e_ms,
        },
        "gpu_launches": len(names) * args.steps,
        "clocks": clocks,
    }
    return result, shape


# ---------------------------------------------------------------------------
# the dense SwiGLU layer (the FFN of the dense layers between the MoE layers)
# ---------------------------------------------------------------------------
DENSE_SHAPES = {   # (T, D, F): the pages give no dense-layer width; F = twice the expert d_ff
    "dense_decode": (16, 5120, 16384),
    "dense_prefill": (8192, 5120, 16384),
}


def run_dense(args, rank: int, world: int, dev: torch.device):
    import int4_quantized_expert_b200 as moe
    T, D, F = DENSE_SHAPES[args.workload]
    g, u, d = (t.to(dev) for t in synth.shared_weights(args.seed, D, F))
    gamma = synth.rms_weight(args.seed, D).to(dev) if args.rmsnorm else None
    layer = moe.DenseLayer(D=D, F=F, w_gate=g, w_up=u, w_down=d, T_max=T, rms_weight=gamma)
    x = synth.tokens(args.seed, T, D).to(dev)
    out = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        layer(x, out)
    torch.cuda.synchronize()
    assert layer.device_status() == moe.Status.OK
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        layer(x, out)
        e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.summary(t0, t1) if sampler else None
    if sampler:
        sampler.stop()
    if layer.device_status() != moe.Status.OK:
        raise RuntimeError("device status after the timed loop")
    ms = max_over_ranks([float(np.mean([a.elapsed_time(b) for a, b in evs]))], dev, world)[0]
    # end to end: pinned host x in, host out, both copies inside the events
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e, e2e_ms = max(3, min(args.steps, 100)), 0.0
    xd = torch.empty_like(x)
    for i in range(n_e2e + 1):
        flush.zero_()
        e0.record(stream)
        xd.copy_(xh, non_blocking=True)
        layer(xd, out)
        oh.copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i > 0:
            e2e_ms += e0.elapsed_time(e1)
    e2e_ms = max_over_ranks([e2e_ms / n_e2e], dev, world)[0]
    hbm_peak, tc_peak, peak_src = peaks()
    wbytes = 3 * D * F * 2
    if T <= 64:   # weight streaming: HBM-bound
        amount = wbytes + T * D * 2 * 2
        roof = {"bound": "hbm", "kernel": "dense layer (all launches)", "achieved": amount / (ms * 1e-3) / 1e9,
                "peak": hbm_peak, "peak_source": peak_src + " copy bandwidth", "unit": "GB/s",
                "traffic": None, "algorithmic_bytes": amount}
    else:
        amount = 2 * T * D * 3 * F
        roof = {"bound": "tensor", "kernel": "dense layer (all launches)", "achieved": amount / (ms * 1e-3) / 1e12,
                "peak": tc_peak, "peak_source": peak_src + " sustained dense bf16", "unit": "TFLOP/s",
                "traffic": None, "algorithmic_flops": amount}
    roof["frac"] = roof["achieved"] / roof["peak"]
    return {
        "metric": METRIC, "value": world * T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded PCG64 x and bf16 weights N(0, 0.02); no dataset)",
        "config": {"workload": "%s: dense SwiGLU FFN layer, T=%d tokens, d_model=%d, d_ff=%d, bf16 weights%s"
                               % (args.workload, T, D, F, ", RMSNorm (eps 1e-5) of x in front" if args.rmsnorm else ""),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "l2": "flushed between steps (256 MB write)"},
        "roofline": roof,
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": T * D * 2,
                "d2h_bytes_per_step": T * D * 2, "ms_per_step": e2e_ms},
        # [rmsnorm,] prep, gate/up, down; the tensor-core path adds the combine
        "gpu_launches": ((3 if T <= 64 else 4) + (1 if args.rmsnorm else 0)) * args.steps,
        "clocks": clocks,
    }


def time_oracle_dense(workload: str, seed: int, budget_s: float, n_steps: int, rms: bool):
    """The oracle's dense layer on single tokens, repeated to fill about
    budget_s per step; returns (tokens/s, sample text, seconds per step)."""
    from oracle import ffn as offn
    T, D, F = DENSE_SHAPES[workload]
    g, u, d = synth.shared_weights(seed, D, F)
    g, u, d = (t.float().numpy().astype(np.float64) for t in (g, u, d))
    gamma = synth.rms_weight(seed, D) if rms else None
    x = synth.tokens(seed, min(T, 64), D)
    t = time.perf_counter()
    offn.dense_forward(x[:1], g, u, d, rms_weight=gamma)
    c1 = max(time.perf_counter() - t, 1e-4)
    n = int(max(1, min(x.shape[0], budget_s / c1)))
    t = time.perf_counter()
    for _ in range(n_steps):
        for i in range(n):
            offn.dense_forward(x[i:i + 1], g, u, d, rms_weight=gamma)
    el = (time.perf_counter() - t) / max(n_steps, 1)
    return n / el, "%d single tokens of %s per step (the full layer for each)" % (n, workload), el


# ---------------------------------------------------------------------------
# the quantize workload (int4_row_quantize of a 16-expert weight set)
# ---------------------------------------------------------------------------
def run_quantize(args, rank: int, world: int, dev: torch.device):
    import int4_quantized_expert_b200 as moe
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed * 1000 + rank)
    mats = []
    for name, rows, cols in quant_matrices(args.experts):
        w = torch.randn(rows, cols, generator=gen, device=dev, dtype=torch.float32).mul_(synth.WEIGHT_STD)
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(rows, cols // args.group_size, dtype=torch.float32, device=dev)
        mats.append((name, w, codes, scales))
    step_bytes = sum(quant_bytes(w.shape[0], w.shape[1], args.group_size) for _, w, _, _ in mats)
    stream = torch.cuda.current_stream()

    def step():
        for _, w, c, sc in mats:
            moe.quantize_int4(w, group_size=args.group_size, out=(c, sc))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for e0, e1 in evs:          # inputs (8 GB) far exceed L2: no flush needed
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.summary(t0, t1) if sampler else None
    if sampler:
        sampler.stop()
    ms = max_over_ranks([float(np.mean([a.elapsed_time(b) for a, b in evs]))], dev, world)[0]

    # end to end: each projection's fp32 weights from pinned host memory, its
    # codes and scales back to pinned host memory, inside the timed region
    host = [(w.cpu().pin_memory(), torch.empty_like(c, device="cpu").pin_memory(),
             torch.empty_like(sc, device="cpu").pin_memory()) for _, w, c, sc in mats]
    n_e2e = max(2, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for i in range(n_e2e + 1):
        e0.record(stream)
        for (_, w, c, sc), (wh, ch, sh) in zip(mats, host):
            w.copy_(wh, non_blocking=True)
            moe.quantize_int4(w, group_size=args.group_size, out=(c, sc))
            ch.copy_(c, non_blocking=True)
            sh.copy_(sc, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i > 0:                # the first pass is a warm-up
            e2e_ms += e0.elapsed_time(e1)
    e2e_ms = max_over_ranks([e2e_ms / n_e2e], dev, world)[0]

    hbm_peak, _, peak_src = peaks()
    achieved = step_bytes / (ms * 1e-3) / 1e9
    h2d = sum(w.numel() * 4 for _, w, _, _ in mats)
    d2h = sum(c.numel() + sc.numel() * 4 for _, _, c, sc in mats)
    result = {
        "metric": QUANT_METRIC,
        "value": world * step_bytes / (ms * 1e-3) / 1e9,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32 -> int4 (fp32 scales)",
        "data": "synthetic (N(0, 0.02) fp32 weights from torch's seeded device generator)",
        "config": {
            "workload": "quantize: int4_row_quantize (group %d) of %d experts x {gate [8192, 5120], " % (
                args.group_size, args.experts) + "up [8192, 5120], down [5120, 8192]} fp32 = %.2f G weights, "
                "3 calls per step" % (args.experts * 3 * 8192 * 5120 / 1e9),
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": "inputs (%.2f GB) larger than L2; no flush" % (args.experts * 3 * 8192 * 5120 * 4 / 1e9),
        },
        "roofline": {"bound": "hbm", "kernel": "quantize_int4", "achieved": achieved, "peak": hbm_peak,
                     "peak_source": peak_src + " copy bandwidth", "unit": "GB/s", "frac": achieved / hbm_peak,
                     "traffic": None, "algorithmic_bytes": step_bytes // len(mats)},
        "e2e": {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": len(mats) * args.steps,
        "clocks": clocks,
    }
    return result


def time_oracle_quantize(seed: int, budget_s: float, n_steps: int, n_warm: int, group: int = 128):
    """The oracle's int4_row_quantize (then packing) on row blocks of the gate
    projection's shape, sized so a step takes about budget_s; returns (GB/s
    of algorithmic bytes, sample text, seconds per step)."""
    from oracle import quant as oq
    w = synth.expert_weights(seed, 0, QUANT_D, QUANT_F)[0]       # [8192, 5120] fp32
    t = time.perf_counter()
    oq.pack_int4(oq.int4_row_quantize(w[:64], group_size=group)[0])
    c64 = max(time.perf_counter() - t, 1e-4)
    rows = int(min(w.shape[0], max(64, budget_s / c64 * 64 // 64 * 64)))
    blk = np.ascontiguousarray(w[:rows])
    for _ in range(n_warm):
        oq.pack_int4(oq.int4_row_quantize(blk, group_size=group)[0])
    t = time.perf_counter()
    for _ in range(n_steps):
        oq.pack_int4(oq.int4_row_quantize(blk, group_size=group)[0])
    el = (time.perf_counter() - t) / max(n_steps, 1)
    sample = ("the first %d of 8192 rows of expert 0's gate projection [8192, 5120] per step (%.2f%% of "
              "the 2.01 G-weight set); GB/s of algorithmic bytes" % (rows, 100.0 * rows * QUANT_D / 2.01e9))
    return quant_bytes(rows, QUANT_D, group) / el / 1e9, sample, el


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------
def oracle_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_layer(shape: synth.LayerShape, seed: int, f_sub: int, token: int, x, group: int = 128):
    """The oracle's layer restricted to the first f_sub hidden units of every
    expert (and of the shared expert): a layer of the same kind whose work per
    token is f_sub / F of the full one.  Weights are quantized before timing."""
    from oracle import ffn as offn, quant as oq, route as oroute
    wr = synth.router_weight(seed, shape.E, shape.D)
    bias = synth.router_bias(shape)
    ids = oroute.route(x[token:token + 1], wr, bias, shape.k)["ids"][0]
    sg, su, sd = synth.shared_weights(seed, shape.D, shape.F_shared)
    fs_sub = max(128, f_sub * shape.F_shared // shape.F // 128 * 128)
    experts = {}
    for e in ids:
        g, u, d = synth.expert_weights(seed, int(e), shape.D, shape.F)
        quant = ((lambda w: oq.int4_row_quantize(w, group_size=group)) if shape.fmt == "int4"
                 else oq.fp8_row_quantize)
        experts[int(e)] = tuple(quant(np.ascontiguousarray(w))
                                for w in (g[:f_sub], u[:f_sub], d[:, :f_sub]))
    return offn.Layer(shape.fmt, shape.k, wr, bias, experts.__getitem__,
                      (sg[:fs_sub], su[:fs_sub], sd[:, :fs_sub].contiguous()), group_size=group), fs_sub


def time_oracle(shape: synth.LayerShape, seed: int, budget_s: float, n_steps: int, n_warm: int,
                group: int = 128):
    """Runs the oracle for one token per step on a hidden-width slice sized so
    a step takes about budget_s; returns (tokens/s, sample text, per-step s)."""
    from oracle import ffn as offn
    x = synth.tokens(seed, shape.T, shape.D)
    probe_f = 128
    lay, fs = oracle_sample_layer(shape, seed, probe_f, 0, x, group)
    t = time.perf_counter()
    offn.moe_forward(lay, x, tokens=[0])
    c128 = max(time.perf_counter() - t, 1e-4)
    f_sub = int(min(shape.F, max(128, (budget_s / c128) * 128 // 128 * 128)))
    lay, fs = oracle_sample_layer(shape, seed, f_sub, 0, x, group)
    for _ in range(n_warm):
        offn.moe_forward(lay, x, tokens=[0])
    t = time.perf_counter()
    for _ in range(n_steps):
        offn.moe_forward(lay, x, tokens=[0])
    el = (time.perf_counter() - t) / max(n_steps, 1)
    frac = f_sub / shape.F
    sample = ("1 token of %s per step, its routed expert(s) and the shared expert restricted to the first "
              "%d of %d (shared %d of %d) hidden units, i.e. %.4f of a token's FFN work; routing over all %d "
              "tokens; tokens/s scaled by that fraction" % (shape.name, f_sub, shape.F, fs, shape.F_shared,
                                                           frac, shape.T))
    return frac / el, sample, el


def run_reference(args):
    budget = min(20.0, 150.0 / max(args.steps + args.warmup, 1))
    if args.workload in DENSE_SHAPES:
        v, sample, per_step = time_oracle_dense(args.workload, args.seed, budget, args.steps, args.rmsnorm)
        T, D, F = DENSE_SHAPES[args.workload]
        return {
            "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded PCG64 x and bf16 weights N(0, 0.02); no dataset)",
            "config": {"workload": "%s: dense SwiGLU FFN layer, T=%d, d_model=%d, d_ff=%d" % (args.workload, T, D, F),
                       "parallelism": "CPU oracle on the host cores"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
    if args.workload == "quantize":
        v, sample, per_step = time_oracle_quantize(args.seed, budget, args.steps, args.warmup, args.group_size)
        return {
            "impl": "reference", "metric": QUANT_METRIC, "value": v, "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 -> int4",
            "data": "synthetic (seeded N(0, 0.02) fp32 weights)",
            "config": {"workload": "quantize (CPU oracle on a row sample)",
                       "parallelism": "CPU oracle on the host cores"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
    shape = synth.SHAPES[args.workload]
    v, sample, per_step = time_oracle(shape, args.seed, budget, args.steps, args.warmup, args.group_size)
    cores = oracle_cores()
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": v,
        "unit": "tokens/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": per_step * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded; no dataset, random-init weights of the stated shapes)",
        "config": {"workload": workload_text(shape, args.group_size), "weights": weights_text(shape, args.group_size),
                   "parallelism": "CPU oracle on the host cores"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="scout_decode",
                    choices=["tiny", "scout_decode", "scout_prefill", "skewed", "maverick_fp8", "maverick_fp8_e16",
                             "quantize", "dense_decode", "dense_prefill"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=QUANT_E,
                    help="quantize workload: experts in the weight set (16; fewer for profiling captures)")
    ap.add_argument("--rmsnorm", action="store_true",
                    help="run the layer with its RMSNorm prologue (gamma ~ 1 + N(0, 0.1), eps 1e-5)")
    ap.add_argument("--group-size", type=int, default=128, choices=[128, 64, 32],
                    help="int4 group size of the routed experts (and of the quantize workload)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    if args.workload in DENSE_SHAPES:
        result = run_dense(args, rank, world, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v, sample, _ = time_oracle_dense(args.workload, args.seed, 10.0, 1, args.rmsnorm)
            result["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
                                      "sample": sample}
    elif args.workload == "quantize":
        result = run_quantize(args, rank, world, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v, sample, _ = time_oracle_quantize(args.seed, budget_s=5.0, n_steps=2, n_warm=0, group=args.group_size)
            result["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": 1,   # element-wise numpy: one thread
                                      "kind": "oracle", "sample": sample}
    else:
        result, shape = run_ours(args, rank, world, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            v, sample, _ = time_oracle(shape, args.seed, budget_s=10.0, n_steps=2, n_warm=0, group=args.group_size)
            result["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": oracle_cores(),
                                      "kind": "oracle", "sample": sample}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
