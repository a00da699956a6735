"""Benchmark of the FP8 linear layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode7b|prefill7b|nested7b|llama70b|small]

A step is one pass of the hot path over one batch of synthetic inputs: for
every (M, shape) layer of the workload, dynamic per-token E4M3 quantisation
of the activations followed by the FP8 GEMM with fused dequantisation
(weights were quantised per output channel once, at set-up, with the same
kernel).  The default workload is the Llama-7B decode linears (QKV
4096->12288, O 4096->4096, gate+up 4096->22016, down 11008->4096 at
M = 1, 4, 8); every layer reads its own weight copy, so one step streams
606 MB of FP8 weights, more than the 126 MB L2, and no weight is L2-resident
when it is read.

Timing: the K timed steps are replayed from a CUDA graph (captured from the
library's own C-ABI calls) between a barrier + synchronize on both sides,
CUDA events on the launching stream, max over ranks.  Per-GEMM durations
for the roofline come from event pairs captured around every GEMM launch of
the last replayed steps.  `e2e` repeats the metric through the public entry
point (fp8_linear_dynamic) with the activations copied from pinned host
memory and the outputs copied back inside the timed region.  `cpu_baseline`
times the CPU oracle on a bounded sample of the same workload.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = None
try:
    with open(os.path.join(ROOT, "BASELINE.json")) as _f:
        METRIC = json.load(_f)["metric"]
except Exception:
    METRIC = "FP8 linear TFLOPS & weight GB/s vs B200 roofline, 7B/70B shapes, M=1–4096"

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOAD_TEXT = {
    "decode7b": "Llama-7B decode linears: QKV 4096->12288, O 4096->4096, gate+up 4096->22016, "
                "down 11008->4096 at M=1,4,8 tokens; dynamic per-token E4M3 activations "
                "(N(0,1), 0.5% x30 outliers), static per-channel E4M3 weights (N(0,0.02)), bf16 out",
    "prefill7b": "Llama-7B prefill linears: same four shapes at M=512,1024,2048; Student-t(4)/sqrt2 "
                 "activations; bf16 out",
    "llama70b": "Llama-70B linears: QKV 8192->10240, O 8192->8192, gate+up 8192->57344, down 28672->8192 "
                "at M=1..4096; Student-t(3) activations; bf16 out",
    "small": "single FP8 linear 16x512x512",
    "nested7b": "NestedFP 7B: 4096->12288 and 11008->4096 at M=1,16,128,1024, FP16 and FP8 modes on the "
                "same hi/lo planes; fp16 out",
}


def _load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- layers
class Layer:
    """One (M, shape, weight copy) layer of a workload."""

    def __init__(self, kind, M, K, N, shape_idx, m_idx, copy):
        self.kind, self.M, self.K, self.N = kind, M, K, N
        self.shape_idx, self.m_idx, self.copy = shape_idx, m_idx, copy

    @property
    def flops(self):
        return 2.0 * self.M * self.N * self.K

    @property
    def weight_bytes(self):
        return self.N * self.K * (2 if self.kind == "nested16" else 1)

    @property
    def gemm_bytes(self):
        """Algorithmic bytes of one GEMM launch: weights once, activations once,
        scales, output once."""
        if self.kind == "fp8":
            return self.N * self.K + self.M * self.K + 4 * self.M + 4 * self.N + 2 * self.M * self.N
        if self.kind == "nested8":
            return self.N * self.K + self.M * self.K + 4 * self.M + 2 * self.M * self.N
        return 2 * self.N * self.K + 2 * self.M * self.K + 2 * self.M * self.N


def workload_layers(name, copies):
    wl = synthetic.WORKLOADS[name]
    layers = []
    if name == "nested7b":
        for mi, M in enumerate(wl.ms):
            for si, (K, N, _) in enumerate(wl.shapes):
                for kind in ("nested16", "nested8"):
                    layers.append(Layer(kind, M, K, N, si, mi, 0))
        return layers
    for mi, M in enumerate(wl.ms):
        for si, (K, N, _) in enumerate(wl.shapes):
            layers.append(Layer("fp8", M, K, N, si, mi, mi % copies))
    return layers


def weight_copies(name):
    # enough distinct weight copies that a step streams more than 3 x L2
    return {"decode7b": 3, "small": 1}.get(name, 1)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="pgf8_clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        load = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- profiled traffic
# The GEMM kernels' sources (and the helpers they include): what a DRAM
# traffic record describes.  The record also names the kernel configuration
# it was taken on.
GEMM_SOURCES = ("gemm.cuh", "gemm_2sm.cuh", "gemm_persistent.cuh", "gemm_streamk.cuh", "quantize.cuh",
                "sm100_ptx.cuh")


def kernel_sources_hash() -> str:
    """Short hash of the GEMM kernels' CUDA sources: profiled counters only
    describe the kernels they were taken on."""
    import hashlib
    csrc = os.path.join(ROOT, "precision_gemm_fp8_b200", "csrc")
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(hashlib.sha256(fh.read()).hexdigest().encode() + b"  " + f.encode() + b"\n")
    return h.hexdigest()[:12]


def profiled_traffic(workload):
    """DRAM bytes (read + write) per launch of the profiled GEMM of this
    workload, from profiles/gemm_traffic.txt, scaled to the workload's average
    launch by algorithmic bytes; None when the kernels changed since the
    capture."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 5 and not line.startswith("#") and parts[0] == workload:
                    src_hash, traffic, algo = parts[1], float(parts[2]), float(parts[3])
                    if src_hash != kernel_sources_hash():
                        return None, "kernels changed since the ncu capture"
                    return traffic, (f"ncu capture of {parts[4]}: DRAM read+write {traffic:.0f} B per launch vs "
                                     f"{algo:.0f} algorithmic B ({traffic / algo:.3f}x)")
    except OSError:
        pass
    return None, "no capture recorded"


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value of x over all ranks (timings are reported as the
    slowest rank's); a no-op for a single process."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank processed units_per_rank units (weak
    scaling, independent replicas), the job took the slowest rank's time."""
    return units_per_rank * world / max_seconds


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import precision_gemm_fp8_b200 as pg

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = _load_peaks()
    name = args.workload
    copies = weight_copies(name)
    layers = workload_layers(name, copies)
    wl = synthetic.WORKLOADS[name]

    # ---- set-up (untimed): weights quantised per channel on the device, activations resident
    weights = {}
    for L in layers:
        key = (L.shape_idx, L.copy, L.kind in ("nested16", "nested8"))
        if key in weights:
            continue
        w = torch.from_numpy(synthetic.weights(name, L.shape_idx, copy=L.copy)).to(dev)
        if key[2]:
            weights[key] = pg.nestedfp_split(w)
        else:
            weights[key] = pg.fp8_quantize_rows(w)
        del w
    acts_host, acts, outs, qbufs = [], [], [], []
    for L in layers:
        x = synthetic.acts(name, L.shape_idx, L.m_idx)
        xh = torch.from_numpy(x).pin_memory()
        acts_host.append(xh)
        acts.append(xh.to(dev))
        out_dt = torch.float16 if L.kind.startswith("nested") else torch.bfloat16
        outs.append(torch.empty((L.M, L.N), dtype=out_dt, device=dev))
        if L.kind == "fp8":
            qbufs.append(torch.zeros(pg.fp8_linear_dynamic_workspace_size(L.M, L.N, L.K), dtype=torch.uint8,
                                     device=dev))
        else:
            mode = pg.NESTED_FP8 if L.kind == "nested8" else pg.NESTED_FP16
            qbufs.append(torch.zeros(max(16, pg.nestedfp_linear_workspace_size(L.M, L.N, L.K, mode)),
                                     dtype=torch.uint8, device=dev))
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    # dynamic layers quantise with their own kernel first (the two-kernel
    # form); with --fused-quant inside the GEMM where the kernel allows it
    xflags = pg.FLAG_FUSED_QUANT if args.fused_quant else 0
    sk_ws = torch.zeros(max(16, max(pg.lib.pgf8_fp8_linear_workspace_size(L.M, L.N, L.K) for L in layers)),
                        dtype=torch.uint8, device=dev)
    # per-tensor activation scaling instead of per-token dynamic (--scaling):
    # one delayed-scaling history or one calibrated amax per layer
    per_tensor = {}
    if args.scaling != "dynamic":
        for i, L in enumerate(layers):
            if L.kind != "fp8":
                continue
            if args.scaling == "delayed":
                per_tensor[i] = pg.DelayedScaling(1024, device=dev)
            else:
                per_tensor[i] = pg.fp8_amax_accumulate(acts[i])   # MINMAX calibration on the layer's input
        torch.cuda.synchronize()

    # --chain: the decoder layer's own producers of each GEMM input: RMSNorm
    # fused with the quantisation ahead of QKV and gate+up, the SiLU gate
    # over the gate+up output fused with the quantisation ahead of down (O
    # keeps its dynamic quantisation: its input is the attention output)
    gammas = {}
    if args.chain:
        if any(L.kind != "fp8" for L in layers) or len(wl.shapes) != 4:
            raise SystemExit("--chain needs a workload of QKV, O, gate+up, down FP8 layers")
        g = torch.Generator().manual_seed(7)
        for i, L in enumerate(layers):
            if L.shape_idx in (0, 2):
                gammas[i] = (0.5 + torch.rand(L.K, generator=g)).to(dev)

    def quantise_chain(i, L, flags):
        aq, sa = pg.dynamic_workspace_views(qbufs[i], L.M, L.K)
        if L.shape_idx in (0, 2):
            pg.fp8_norm_quantize(acts[i], gammas[i], None, 1e-6, aq, sa, flags=flags, stream=stream)
        elif L.shape_idx == 3:
            pg.fp8_silu_mul_quantize(outs[i - 1], aq, sa, flags=flags, stream=stream)
        else:
            pg.fp8_quantize_rows(acts[i], aq, sa, stream=stream)
        return aq, sa

    def quantise_per_tensor(i, L, flags=0):
        aq, sa = pg.dynamic_workspace_views(qbufs[i], L.M, L.K)
        if args.scaling == "delayed":
            per_tensor[i].step(acts[i], aq, sa, flags=flags, stream=stream)
        else:
            pg.fp8_quantize_tensor(acts[i], per_tensor[i], aq, sa, flags=flags, stream=stream)
        return aq, sa

    def enqueue_step(ev_pairs=None):
        """One step through the C ABI on `stream`.

        Without ev_pairs: the layers are chained as in inference — every call
        carries FLAG_OVERLAP_PREVIOUS, so each layer's quantisation and weight
        loads overlap the previous layer's tail (programmatic dependent
        launch).  With ev_pairs: the same kernels through the two-call form,
        an event pair bracketing every GEMM launch (each GEMM then runs in
        isolation; these are the durations the roofline uses)."""
        for i, L in enumerate(layers):
            W = weights[(L.shape_idx, L.copy, L.kind != "fp8")]
            if L.kind == "fp8" and args.chain:
                if ev_pairs is None and L.shape_idx == 1:   # O: the dynamic pair, overlapped
                    pg.fp8_linear_dynamic(acts[i], W[0], W[1], y=outs[i], workspace=qbufs[i],
                                          flags=pg.FLAG_OVERLAP_PREVIOUS, stream=stream)
                    continue
                if ev_pairs is None:
                    aq, sa = quantise_chain(i, L, pg.FLAG_OVERLAP_PREVIOUS)
                    pg.fp8_linear(aq, sa, W[0], W[1], y=outs[i], workspace=sk_ws, flags=pg.FLAG_OVERLAP_PREVIOUS,
                                  stream=stream)
                    continue
                ev_pairs[i][2].record(stream)
                aq, sa = quantise_chain(i, L, 0)
                ev_pairs[i][0].record(stream)
                pg.fp8_linear(aq, sa, W[0], W[1], y=outs[i], workspace=sk_ws, stream=stream)
                ev_pairs[i][1].record(stream)
                continue
            if L.kind == "fp8":
                if ev_pairs is None and not per_tensor:
                    pg.fp8_linear_dynamic(acts[i], W[0], W[1], y=outs[i], workspace=qbufs[i],
                                          flags=pg.FLAG_OVERLAP_PREVIOUS | xflags, stream=stream)
                    continue
                if ev_pairs is None:
                    aq, sa = quantise_per_tensor(i, L, pg.FLAG_OVERLAP_PREVIOUS)
                    pg.fp8_linear(aq, sa, W[0], W[1], y=outs[i], workspace=sk_ws, flags=pg.FLAG_OVERLAP_PREVIOUS,
                                  stream=stream)
                    continue
                ev_pairs[i][2].record(stream)
                if per_tensor:
                    aq, sa = quantise_per_tensor(i, L)
                else:
                    aq, sa = pg.dynamic_workspace_views(qbufs[i], L.M, L.K)
                    pg.fp8_quantize_rows(acts[i], aq, sa, stream=stream)
                ev_pairs[i][0].record(stream)
                pg.fp8_linear(aq, sa, W[0], W[1], y=outs[i], workspace=sk_ws, stream=stream)
                ev_pairs[i][1].record(stream)
            else:
                mode = pg.NESTED_FP16 if L.kind == "nested16" else pg.NESTED_FP8
                if ev_pairs is not None:
                    ev_pairs[i][0].record(stream)
                pg.nestedfp_linear(acts[i], W[0], W[1] if mode == pg.NESTED_FP16 else None, mode=mode,
                                   y=outs[i], workspace=qbufs[i],
                                   flags=xflags if ev_pairs is not None else pg.FLAG_OVERLAP_PREVIOUS | xflags,
                                   stream=stream)
                if ev_pairs is not None:
                    ev_pairs[i][1].record(stream)

    launches_per_step = sum(2 if L.kind in ("fp8", "nested8") else 1 for L in layers)

    # ---- graph of R steps (R-1 chained, the last with per-GEMM events), replayed K / R times
    K, W = args.steps, args.warmup
    R = max(1, min(10, K))
    while K % R:
        R -= 1
    evs = [tuple(torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)) for _ in layers]
    with torch.cuda.stream(stream):
        enqueue_step()          # load modules / first-call set-up outside capture
        enqueue_step(evs)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for r in range(R):
            enqueue_step(evs if r == R - 1 else None)
    with torch.cuda.stream(stream):
        for _ in range(max(1, W // R)):
            graph.replay()
    torch.cuda.synchronize()
    if pg.device_status(stream) != pg.OK:
        raise RuntimeError("device error word raised during warm-up")

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    sampler = ClockSampler(local_rank)
    sampler.start()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(K // R):
            graph.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, dev)
    st = pg.device_status(stream)
    if st != pg.OK:
        raise RuntimeError(f"device error word raised in the timed region: {st}")

    # per-GEMM durations (ms) from the event-bracketed step of the last replay
    per_layer_ms = np.array([evs[i][0].elapsed_time(evs[i][1]) for i in range(len(layers))])
    quant_ms = np.array([evs[i][2].elapsed_time(evs[i][0]) if L.kind == "fp8" else 0.0
                         for i, L in enumerate(layers)])

    ms_step = ms_total / K
    wbytes = sum(L.weight_bytes for L in layers)
    flops = sum(L.flops for L in layers)
    gbs = job_throughput(wbytes / 1e9, world, ms_step * 1e-3)        # whole job, all ranks
    tflops = job_throughput(flops / 1e12, world, ms_step * 1e-3)

    # roofline of the dominant kernel (the GEMM)
    gemm_bytes = sum(L.gemm_bytes for L in layers)
    gemm_flops = sum(L.flops for L in layers)
    gemm_time_s = per_layer_ms.sum() * 1e-3
    memory_bound = name in ("decode7b", "small")
    if memory_bound:
        achieved = gemm_bytes / gemm_time_s / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": None,
                "peak_source": f"{peak_src} HBM copy bandwidth"}
    else:
        # The GEMMs are timed inside a long, power-capped step: the sustained
        # bf16 figure is the denominator (x 2, the FP8 / bf16 nominal ratio);
        # the fraction of the burst figure is reported beside it.
        achieved = gemm_flops / gemm_time_s / 1e12
        sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
        peak = 2.0 * sustained
        burst = 2.0 * float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": None,
                "peak_source": f"{peak_src} bf16 sustained x 2 (FP8 nominal ratio); kernels timed inside a "
                               f"long power-capped step",
                "frac_of_burst_peak": round(achieved / burst, 4), "burst_peak": burst}
    roof["kernel"] = "pgf8::gemm_kernel"
    roof["launches_timed"] = int(len(layers))
    # share of the GEMM among this step's kernels, each timed alone (the
    # figure to compare with the ncu launch list, which also serialises)
    roof["gemm_share_of_kernel_time"] = round(float(per_layer_ms.sum()) /
                                              float(per_layer_ms.sum() + quant_ms.sum()), 3)
    roof["gemm_isolated_sum_over_chained_step"] = round(float(per_layer_ms.sum()) / ms_step, 3)
    roof["traffic"], roof["traffic_note"] = profiled_traffic(name)

    per_layer = []
    for L, t in zip(layers, per_layer_ms):
        per_layer.append({"kind": L.kind, "M": L.M, "K": L.K, "N": L.N, "us": round(t * 1e3, 2),
                          "gbs": round(L.gemm_bytes / (t * 1e-3) / 1e9, 1),
                          "tflops": round(L.flops / (t * 1e-3) / 1e12, 1)})

    # ---- e2e through the public entry point, host buffers, copies inside the timed region
    e2e = run_e2e(pg, torch, dev, layers, weights, acts_host, outs, args, world, wbytes, flops, memory_bound)

    result = {
        "metric": METRIC,
        "value": round(gbs if memory_bound else tflops, 2),
        "unit": "GB/s" if memory_bound else "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8e4m3" if name != "nested7b" else "fp16+fp8e4m3/e5m2",
        "data": "synthetic",
        "config": {"workload": f"{name}: {WORKLOAD_TEXT[name]}",
                   "l2": "inputs larger than L2 (%d weight copies; %.0f MB of weights streamed per step)"
                         % (copies, wbytes / 1e6),
                   "timing": "CUDA graph of the C-ABI calls (R-1 chained steps + 1 event-bracketed step), "
                             "replayed K/R times, R=%d" % R,
                   "quantisation": "inside the skinny GEMM where each CTA's activation slice fits its "
                                   "registers, else its own kernel" if args.fused_quant
                   else "own kernel before each GEMM",
                   "chain": ("decoder layer: RMSNorm+quantise -> QKV; quantise -> O; RMSNorm+quantise -> "
                             "gate+up; SiLU gate+quantise of the gate+up output -> down") if args.chain else None,
                   "activation_scaling": {"dynamic": "per token, dynamic",
                                          "delayed": "per tensor, delayed (amax history of 1024 per layer)",
                                          "static": "per tensor, MINMAX-calibrated amax"}[args.scaling]},
        "secondary": {"tflops": round(tflops, 3), "weight_gbs": round(gbs, 1)},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * K),
        "clocks": clocks,
        "per_layer": per_layer,
    }
    return result


def run_e2e(pg, torch, dev, layers, weights, acts_host, outs, args, world, wbytes, flops, memory_bound):
    """The metric end to end through the public API with host buffers: every
    step copies all of its activations from one pinned host buffer to the
    device, runs the layers (one pgf8_fp8_linear_dynamic_many call for the
    FP8 workloads, one nestedfp_linear call per layer otherwise) and copies
    all outputs back to one pinned host buffer; the copies are inside the
    timed region."""
    stream = torch.cuda.Stream(device=dev)
    # packed activations / outputs (16-byte aligned slices)
    def packed(tensors, device):
        offs, total = [], 0
        for t in tensors:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        buf = torch.empty(total, dtype=torch.uint8, device=device, pin_memory=(device == "cpu"))
        views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, tensors)]
        return buf, views
    x_host, x_host_views = packed(acts_host, "cpu")
    for v, a in zip(x_host_views, acts_host):
        v.copy_(a)
    x_dev, x_views = packed(acts_host, dev)
    y_dev, y_views = packed(outs, dev)
    y_host, _ = packed(outs, "cpu")
    ws = []
    for L in layers:
        if L.kind == "fp8":
            ws.append(torch.zeros(pg.fp8_linear_dynamic_workspace_size(L.M, L.N, L.K), dtype=torch.uint8,
                                  device=dev))
        else:
            mode = pg.NESTED_FP8 if L.kind == "nested8" else pg.NESTED_FP16
            ws.append(torch.zeros(max(16, pg.nestedfp_linear_workspace_size(L.M, L.N, L.K, mode)),
                                  dtype=torch.uint8, device=dev))
    all_fp8 = all(L.kind == "fp8" for L in layers)
    seq = None
    per_tensor = {}
    gammas = {}
    if all_fp8 and args.chain:
        g = torch.Generator().manual_seed(7)
        for i, L in enumerate(layers):
            if L.shape_idx in (0, 2):
                gammas[i] = (0.5 + torch.rand(L.K, generator=g)).to(dev)
    elif all_fp8 and args.scaling != "dynamic":
        for i, L in enumerate(layers):
            per_tensor[i] = (pg.DelayedScaling(1024, device=dev) if args.scaling == "delayed"
                             else pg.fp8_amax_accumulate(x_views[i].copy_(acts_host[i].to(dev))))
        torch.cuda.synchronize()
    elif all_fp8:
        seq = pg.LayerSequence([(x_views[i], weights[(L.shape_idx, L.copy, False)][0],
                                 weights[(L.shape_idx, L.copy, False)][1], y_views[i], ws[i])
                                for i, L in enumerate(layers)])

    def step():
        with torch.cuda.stream(stream):
            x_dev.copy_(x_host, non_blocking=True)
            if seq is not None:
                seq.run(flags=pg.FLAG_FUSED_QUANT if args.fused_quant else 0, stream=stream)
            elif gammas:
                for i, L in enumerate(layers):
                    W = weights[(L.shape_idx, L.copy, False)]
                    aq, sa = pg.dynamic_workspace_views(ws[i], L.M, L.K)
                    fl = pg.FLAG_OVERLAP_PREVIOUS if i else 0
                    if L.shape_idx == 1:
                        pg.fp8_linear_dynamic(x_views[i], W[0], W[1], y=y_views[i], workspace=ws[i], flags=fl,
                                              stream=stream)
                        continue
                    if L.shape_idx in (0, 2):
                        pg.fp8_norm_quantize(x_views[i], gammas[i], None, 1e-6, aq, sa, flags=fl, stream=stream)
                    else:
                        pg.fp8_silu_mul_quantize(y_views[i - 1], aq, sa, flags=fl, stream=stream)
                    pg.fp8_linear(aq, sa, W[0], W[1], y=y_views[i], workspace=ws[i],
                                  flags=pg.FLAG_OVERLAP_PREVIOUS, stream=stream)
            elif per_tensor:
                for i, L in enumerate(layers):
                    W = weights[(L.shape_idx, L.copy, False)]
                    aq, sa = pg.dynamic_workspace_views(ws[i], L.M, L.K)
                    fl = pg.FLAG_OVERLAP_PREVIOUS if i else 0
                    if args.scaling == "delayed":
                        per_tensor[i].step(x_views[i], aq, sa, flags=fl, stream=stream)
                    else:
                        pg.fp8_quantize_tensor(x_views[i], per_tensor[i], aq, sa, flags=fl, stream=stream)
                    pg.fp8_linear(aq, sa, W[0], W[1], y=y_views[i], workspace=ws[i],
                                  flags=pg.FLAG_OVERLAP_PREVIOUS, stream=stream)
            else:
                for i, L in enumerate(layers):
                    W = weights[(L.shape_idx, L.copy, True)]
                    mode = pg.NESTED_FP16 if L.kind == "nested16" else pg.NESTED_FP8
                    fl = (pg.FLAG_OVERLAP_PREVIOUS if i else 0) | (pg.FLAG_FUSED_QUANT if args.fused_quant else 0)
                    pg.nestedfp_linear(x_views[i], W[0], W[1] if mode == pg.NESTED_FP16 else None, mode=mode,
                                       y=y_views[i], workspace=ws[i], flags=fl, stream=stream)
            y_host.copy_(y_dev, non_blocking=True)

    steps = max(3, min(args.steps, 200))
    for _ in range(3):
        step()
    stream.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    stream.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    h2d = int(x_host.numel())
    d2h = int(y_host.numel())
    v = job_throughput(wbytes / 1e9 if memory_bound else flops / 1e12, world, ms * 1e-3)
    return {"value": round(v, 2), "unit": "GB/s" if memory_bound else "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms, 5),
            "entry_point": ("pgf8_nestedfp_linear" if not all_fp8 else
                            "pgf8_fp8_norm_quantize / pgf8_fp8_silu_mul_quantize / pgf8_fp8_quantize_rows + "
                            "pgf8_fp8_linear per layer" if args.chain else "pgf8_fp8_linear_dynamic_many"
                            if args.scaling == "dynamic" else
                            {"delayed": "pgf8_fp8_quantize_delayed", "static": "pgf8_fp8_quantize_tensor"}[args.scaling]
                            + " + pgf8_fp8_linear per layer")}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(name, cols):
    """Time the CPU oracle on every layer of one step of the workload: the
    activations are quantised in full, the binary64 contraction runs on the
    first `cols` output channels of each layer, and its time is extrapolated
    linearly to all N channels.  Returns (seconds per full step, description,
    threads used)."""
    import oracle

    layers = workload_layers(name, weight_copies(name))
    total = 0.0
    for L in layers:
        x = synthetic.acts(name, L.shape_idx, L.m_idx)
        ncols = min(cols, L.N)
        w = synthetic.weights(name, L.shape_idx, copy=L.copy, n_override=ncols)
        if L.kind == "fp8":
            wq, sw = oracle.quantize_rows(w)      # offline weight quantisation: not timed
            t0 = time.perf_counter()
            aq, sa = oracle.quantize_rows(x)
            t1 = time.perf_counter()
            oracle.fp8_linear(aq, sa, wq, sw)
        elif L.kind == "nested16":
            hi, lo = oracle.nestedfp_split(w)
            t0 = t1 = time.perf_counter()
            oracle.nestedfp_linear_fp16(x, hi, lo)
        else:
            hi, _ = oracle.nestedfp_split(w)
            t0 = t1 = time.perf_counter()
            oracle.nestedfp_linear_fp8(x, hi)
        t2 = time.perf_counter()
        total += (t1 - t0) + (t2 - t1) * (L.N / ncols)
    desc = (f"all {len(layers)} layers of one step: activations quantised in full, binary64 contraction on "
            f"the first {cols} output channels of each layer, its time scaled linearly to all N channels")
    return total, desc, 1


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores; each
    step is a bounded sample of one step of the workload (a number of output
    channels per layer sized so the whole --steps/--warmup run takes about two
    minutes), extrapolated to the full step."""
    name = args.workload
    layers = workload_layers(name, weight_copies(name))
    wbytes = sum(L.weight_bytes for L in layers)
    flops = sum(L.flops for L in layers)
    memory_bound = name in ("decode7b", "small")
    # size the per-step sample so the whole run takes about two minutes
    t_start = time.perf_counter()
    oracle_sample(name, cols=8)
    t8 = time.perf_counter() - t_start
    budget = max(0.02, 120.0 / (args.warmup + args.steps))
    cols = int(max(1, min(4096, 8 * budget / max(t8, 1e-6))))
    times = []
    desc = ""
    for i in range(args.warmup + args.steps):
        s, desc, _ = oracle_sample(name, cols=cols)
        if i >= args.warmup:
            times.append(s)
    ms = 1e3 * sum(times) / len(times)
    v = (wbytes / (ms * 1e-3) / 1e9) if memory_bound else (flops / (ms * 1e-3) / 1e12)
    unit = "GB/s" if memory_bound else "TFLOP/s"
    return {
        "metric": METRIC, "value": v, "unit": unit, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{name}: {WORKLOAD_TEXT[name]}"},
        "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": desc, "value": v, "unit": unit},
        "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main
def run_single(args):
    """One layer, launched eagerly `warmup + steps` times: the small, fixed case
    the profiler captures (e.g. --single fp8,8,4096,12288 = kind,M,K,N)."""
    import torch
    import precision_gemm_fp8_b200 as pg

    kind, M, K, N = args.single.split(",")
    M, K, N = int(M), int(K), int(N)
    dev = torch.device("cuda", 0)
    g = synthetic.rng(99, 0, 0, 0)
    w = torch.from_numpy(synthetic.weights_f16(N, K, 0.02, g)).to(dev)
    x = torch.from_numpy(synthetic.activations("normal_outl_0p5pct_x30", M, K, g)).to(dev)
    opts = dict(path=args.path, split_k=args.split_k, tile_n=args.tile_n)
    if kind == "fp8":
        wq, sw = pg.fp8_quantize_rows(w)
        aq, sa = pg.fp8_quantize_rows(x)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        fn = lambda: pg.fp8_linear(aq, sa, wq, sw, y=y, **opts)  # noqa: E731
    elif kind == "dyn":
        wq, sw = pg.fp8_quantize_rows(w)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=dev)
        fn = lambda: pg.fp8_linear_dynamic(x, wq, sw, y=y, workspace=ws, **opts)  # noqa: E731
    else:
        hi, lo = pg.nestedfp_split(w.half())
        x16 = x.half()
        mode = pg.NESTED_FP16 if kind == "nested16" else pg.NESTED_FP8
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        ws = torch.zeros(max(16, pg.nestedfp_linear_workspace_size(M, N, K, mode)), dtype=torch.uint8, device=dev)
        fn = lambda: pg.nestedfp_linear(x16, hi, lo, mode=mode, y=y, workspace=ws, **opts)  # noqa: E731
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    if pg.device_status() != pg.OK:
        raise RuntimeError("device error word raised")
    us = 1e3 * t0.elapsed_time(t1) / args.steps
    print(json.dumps({"single": args.single, "us_per_call": round(us, 3), "opts": opts,
                      "weight_gbs": round(N * K * (2 if kind == "nested16" else 1) / (us * 1e-6) / 1e9, 1),
                      "tflops": round(2.0 * M * N * K / (us * 1e-6) / 1e12, 2)}), flush=True)


def run_attention(args):
    """Decode attention over the FP8 paged cache, launched eagerly `warmup +
    steps` times (e.g. --attention 64,64,8,128,4096 = seqs, query heads, KV
    heads, head_dim, context: a 70B-shaped decode batch).  Caches of
    N(0,1) K / V written by the cache writer with per-head scales 4.5/448,
    blocks of 16 positions scattered by a seeded permutation; the caches
    (2 x seqs x context x KV heads x head_dim bytes) exceed L2 at the
    intended sizes, so every call streams them from HBM."""
    import torch
    import precision_gemm_fp8_b200 as pg

    seqs, hq, hkv, d, ctx = (int(v) for v in args.attention.split(","))
    B = 16
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    nblk = (ctx + B - 1) // B
    num_blocks = seqs * nblk
    tables = torch.randperm(num_blocks, generator=gen, device=dev).to(torch.int32).view(seqs, nblk)
    kc = torch.zeros((num_blocks, hkv, B, d), dtype=torch.uint8, device=dev)
    vc = torch.zeros_like(kc)
    sk = torch.full((hkv,), 4.5 / 448.0, dtype=torch.float32, device=dev)
    sv = sk.clone()
    for s in range(seqs):
        for cache, sc in ((kc, sk), (vc, sv)):
            kv = torch.randn((ctx, hkv, d), generator=gen, device=dev)
            pg.fp8_kv_write_paged(kv, sc, cache, tables[s].contiguous(), 0)
    q = torch.randn((seqs, hq, d), generator=gen, device=dev)
    lens = torch.full((seqs,), ctx, dtype=torch.int32, device=dev)
    out = torch.empty((seqs, hq, d), dtype=torch.float32, device=dev)
    nsplit, chunk = pg.fp8_attention_decode_plan(seqs, hq, hkv, d, ctx, args.split_k)
    ws_bytes = pg.lib.pgf8_fp8_attention_decode_workspace_size(seqs, hq, hkv, d, ctx, args.split_k)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    flags = pg.FLAG_ATTN_MMA if args.attn_mma else 0
    fn = lambda: pg.fp8_attention_decode_paged(q, kc, vc, sk, sv, tables, lens, ctx, out=out,  # noqa: E731
                                               splits=args.split_k, workspace=ws, flags=flags)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    if pg.device_status() != pg.OK:
        raise RuntimeError("device error word raised")
    us = 1e3 * t0.elapsed_time(t1) / args.steps
    kv_bytes = 2 * seqs * ctx * hkv * d
    alg = kv_bytes + seqs * hq * d * 8 + seqs * nblk * 4
    peaks, src = _load_peaks()
    gbs = alg / (us * 1e-6) / 1e9
    print(json.dumps({"attention": args.attention, "tensor_cores": bool(args.attn_mma), "us_per_call": round(us, 3),
                      "nsplit": nsplit, "chunk": chunk,
                      "algorithmic_bytes": alg, "kv_bytes": kv_bytes, "gbs": round(gbs, 1),
                      "frac_hbm": round(gbs / float(peaks["hbm_gbs"]), 3), "peak_source": src}), flush=True)


def run_kv_write(args):
    """The FP8 paged KV-cache writer, launched eagerly `warmup + steps` times
    (e.g. --kv-write 2048,32,128 = tokens, KV heads, head_dim: one 7B
    prefill's K).  The K rows are a bf16 slice of a QKV-projection-shaped
    output [tokens, (32 + 2 * heads) * head_dim] read in place; positions
    0 .. tokens - 1 through a seeded permutation of blocks of 16."""
    import torch
    import precision_gemm_fp8_b200 as pg

    tokens, heads, d = (int(v) for v in args.kv_write.split(","))
    B = 16
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    width = (32 + 2 * heads) * d
    qkv = torch.randn((tokens, width), generator=gen, device=dev).to(torch.bfloat16)
    k = torch.as_strided(qkv, (tokens, heads, d), (width, d, 1), 32 * d)
    nblk = (tokens + B - 1) // B
    table = torch.randperm(nblk, generator=gen, device=dev).to(torch.int32)
    cache = torch.zeros((nblk, heads, B, d), dtype=torch.uint8, device=dev)
    scales = torch.full((heads,), 4.5 / 448.0, dtype=torch.float32, device=dev)
    fn = lambda: pg.fp8_kv_write_paged(k, scales, cache, table, 0)  # noqa: E731
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    if pg.device_status() != pg.OK:
        raise RuntimeError("device error word raised")
    us = 1e3 * t0.elapsed_time(t1) / args.steps
    alg = tokens * heads * d * 3 + nblk * 4      # bf16 in, E4M3 out, the table
    peaks, src = _load_peaks()
    gbs = alg / (us * 1e-6) / 1e9
    print(json.dumps({"kv_write": args.kv_write, "us_per_call": round(us, 3), "algorithmic_bytes": alg,
                      "gbs": round(gbs, 1), "frac_hbm": round(gbs / float(peaks["hbm_gbs"]), 3),
                      "peak_source": src, "l2_note": "inputs below L2 size are timed warm"}), flush=True)


def run_attention_context(args):
    """Context attention over the FP8 paged cache, launched eagerly `warmup +
    steps` times (e.g. --attention-context 4,32,32,2048 = seqs, query heads,
    KV heads, prompt length: 7B-shaped prefill, each sequence's prompt is its
    whole context).  Queries N(0,1) quantised per (token, head) row by the
    row quantiser before the timed region; caches as for --attention.
    FLOPs counted: 4 * 128 * sum over query rows of the keys they see (the
    causal half of Q K^T and P V), per query head."""
    import torch
    import precision_gemm_fp8_b200 as pg

    seqs, hq, hkv, qlen = (int(v) for v in args.attention_context.split(","))
    d, B, ctx = 128, 16, qlen
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321)
    nblk = (ctx + B - 1) // B
    num_blocks = seqs * nblk
    tables = torch.randperm(num_blocks, generator=gen, device=dev).to(torch.int32).view(seqs, nblk)
    kc = torch.zeros((num_blocks, hkv, B, d), dtype=torch.uint8, device=dev)
    vc = torch.zeros_like(kc)
    sk = torch.full((hkv,), 4.5 / 448.0, dtype=torch.float32, device=dev)
    sv = sk.clone()
    for s in range(seqs):
        for cache, sc in ((kc, sk), (vc, sv)):
            kv = torch.randn((ctx, hkv, d), generator=gen, device=dev)
            pg.fp8_kv_write_paged(kv, sc, cache, tables[s].contiguous(), 0)
    total_q = seqs * qlen
    q = torch.randn((total_q * hq, d), generator=gen, device=dev)
    qc, qs = pg.fp8_quantize_rows(q)
    qc = qc.view(total_q, hq, d)
    q_start = torch.arange(0, total_q + 1, qlen, dtype=torch.int32, device=dev)
    lens = torch.full((seqs,), ctx, dtype=torch.int32, device=dev)
    out = torch.empty((total_q, hq, d), dtype=torch.bfloat16, device=dev)
    fn = lambda: pg.fp8_attention_context_paged(qc, qs, q_start, lens, kc, vc, sk, sv, tables, ctx, qlen,  # noqa: E731
                                                out=out)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    if pg.device_status() != pg.OK:
        raise RuntimeError("device error word raised")
    us = 1e3 * t0.elapsed_time(t1) / args.steps
    seen = qlen * (qlen + 1) // 2          # keys seen, summed over the query rows of one sequence
    flops = 4.0 * d * seen * hq * seqs
    peaks, src = _load_peaks()
    fp8_peak = 2.0 * float(peaks["bf16_tflops"])
    tf = flops / (us * 1e-6) / 1e12
    print(json.dumps({"attention_context": args.attention_context, "us_per_call": round(us, 3),
                      "flops": flops, "tflops": round(tf, 1), "frac_fp8_burst": round(tf / fp8_peak, 3),
                      "fp8_peak_tflops": fp8_peak, "peak_source": src}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(synthetic.WORKLOADS), default="decode7b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scaling", choices=["dynamic", "delayed", "static"], default="dynamic",
                    help="activation scales of the FP8 layers: per-token dynamic (default), per-tensor delayed "
                         "(amax history of 1024) or per-tensor static (MINMAX-calibrated)")
    ap.add_argument("--chain", action="store_true",
                    help="feed each GEMM from its decoder-layer producer: RMSNorm fused with the quantisation ahead "
                         "of QKV and gate+up, the SiLU gate of the gate+up output ahead of down")
    ap.add_argument("--fused-quant", action="store_true",
                    help="quantise dynamic activations inside the skinny GEMM where its kernel allows it")
    ap.add_argument("--single", default=None, help="kind,M,K,N: time (or profile) one layer eagerly")
    ap.add_argument("--attention", default=None,
                    help="seqs,q_heads,kv_heads,head_dim,context: time (or profile) the FP8 paged decode attention "
                         "eagerly (--split-k caps its context chunks)")
    ap.add_argument("--attn-mma", action="store_true",
                    help="with --attention: both products on the tensor cores (PGF8_FLAG_ATTN_MMA)")
    ap.add_argument("--attention-context", default=None,
                    help="seqs,q_heads,kv_heads,prompt_len: time (or profile) the FP8 paged context attention "
                         "eagerly (head_dim 128, causal prompts)")
    ap.add_argument("--kv-write", default=None,
                    help="tokens,kv_heads,head_dim: time (or profile) the FP8 paged KV-cache writer eagerly")
    ap.add_argument("--path", type=int, default=0)
    ap.add_argument("--split-k", type=int, default=0)
    ap.add_argument("--tile-n", type=int, default=0)
    args = ap.parse_args()
    if args.chain and (args.scaling != "dynamic" or args.fused_quant):
        ap.error("--chain measures the decoder-layer producers with per-token scales; it takes neither "
                 "--scaling nor --fused-quant")
    if args.single:
        run_single(args)
        return
    if args.attention:
        run_attention(args)
        return
    if args.attention_context:
        run_attention_context(args)
        return
    if args.kv_write:
        run_kv_write(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:      # the other ranks exit without work
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if not args.no_cpu_baseline:
                s, desc, cores = oracle_sample(args.workload, cols=1024)
                layers = workload_layers(args.workload, weight_copies(args.workload))
                wbytes = sum(L.weight_bytes for L in layers)
                flops = sum(L.flops for L in layers)
                v = (wbytes / s / 1e9) if res["unit"] == "GB/s" else (flops / s / 1e12)
                res["cpu_baseline"] = {"value": v, "unit": res["unit"], "cores": cores, "kind": "oracle",
                                       "sample": desc, "ms_per_step_extrapolated": round(s * 1e3, 1),
                                       "host_cpus": os.cpu_count()}
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
