"""Benchmark of the FP8 linear layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama70b|decode7b|prefill7b|nested7b|small] [--per-layer]

A step is one pass of the hot path over one batch of synthetic inputs: for
every (M, shape) layer of the workload, dynamic per-token E4M3 quantisation
of the activations followed by the FP8 GEMM with fused dequantisation
(weights were quantised per output channel once, at set-up, with the same
kernel).  The default workload is the Llama-70B linears (QKV 8192->10240,
O 8192->8192, gate+up 8192->57344, down 28672->8192) at M = 1, 2, 4, ...,
4096 tokens: 52 independent layers, 11.1 GB of FP8 weights streamed per step
(the same weights for every M, 855 MB per M: more than the 126 MB L2, so no
weight is L2-resident when it is re-read).  One step is one
pgf8_fp8_linear_dynamic_group call: the M <= 256 layers stream their weights
through the grouped kernel, the larger ones run the tiled tensor-core GEMMs.
decode7b, prefill7b and nested7b are timed as secondary steps in the same run.

Timing: the K timed steps are replayed from a CUDA graph (captured from the
library's own C-ABI calls) between a barrier + synchronize on both sides,
CUDA events on the launching stream, max over ranks.  The per-kernel shares
for the roofline come from a step run with an event between consecutive
launch groups, scaled to the timed step.  `e2e` repeats the metric through
the public entry point with the activations copied from pinned host memory
and the outputs copied back inside the timed region.  `cpu_baseline` times
the CPU oracle on a bounded sample of the same workload, one thread and all
host threads.

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
                "same hi/lo planes (3 weight copies, one per M but M=1024 sharing the M=1 copy); fp16 out",
    "nested7b_decode": "NestedFP 7B decode: the nested7b shapes at its decode sizes M=1,16, three times each, "
                       "every (repeat, M) with its own weight copy (6 copies: no re-read from L2), FP16 and FP8 "
                       "modes; fp16 out",
}

# bench-only workloads: a subset of a seeded workload's layers (same inputs)
BASE_WORKLOAD = {"nested7b_decode": "nested7b"}


def base_workload(name):
    return BASE_WORKLOAD.get(name, name)


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
    wl = synthetic.WORKLOADS[base_workload(name)]
    layers = []
    if name == "nested7b":
        for mi, M in enumerate(wl.ms):
            for si, (K, N, _) in enumerate(wl.shapes):
                for kind in ("nested16", "nested8"):
                    layers.append(Layer(kind, M, K, N, si, mi, mi % copies))
        return layers
    if name == "nested7b_decode":
        # every (repeat, M) its own weight copy: no layer re-reads planes an
        # earlier layer of its group left in L2
        dec = [(mi, M) for mi, M in enumerate(wl.ms) if M <= 16]
        for c in range(copies):
            mi, M = dec[c % len(dec)]
            for si, (K, N, _) in enumerate(wl.shapes):
                for kind in ("nested16", "nested8"):
                    layers.append(Layer(kind, M, K, N, si, mi, c))
        return layers
    for mi, M in enumerate(wl.ms):
        for si, (K, N, _) in enumerate(wl.shapes):
            layers.append(Layer("fp8", M, K, N, si, mi, mi % copies))
    return layers


def weight_copies(name):
    # enough distinct weight copies that a step streams more than 3 x L2
    return {"decode7b": 3, "nested7b": 3, "nested7b_decode": 6, "small": 1}.get(name, 1)


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
# The sources of the kernels the recorded FP8 steps run (and the helpers
# they include): what a DRAM traffic record describes.  The record also
# names the kernel configuration it was taken on.  (The NestedFP-only
# swapped FP16 kernel, gemm_persistent_swap.cuh, runs in none of them.)
GEMM_SOURCES = ("gemm.cuh", "gemm_2sm.cuh", "gemm_pair_group.cuh", "gemm_persistent.cuh", "gemm_streamk.cuh", "gemm_group.cuh",
                "quantize.cuh", "sm100_ptx.cuh")


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
def measure_fp8_peak(torch, dev, seconds=2.0):
    """Dense E4M3 GEMM throughput of the installed library (torch._scaled_mm,
    8192^3, bf16 out, per-tensor unit scales): best of 10 single calls
    (burst) and the mean of back-to-back calls over `seconds` (sustained,
    power-capped).  Library timing, used only as a reference figure."""
    n = 8192
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        fn = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)  # noqa: E731
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        reps = max(10, int(seconds * 1e3 / best))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        e1.synchronize()
        mean = e0.elapsed_time(e1) / reps
        flops = 2.0 * n ** 3
        del a, b
        return {"burst_tflops": round(flops / (best * 1e-3) / 1e12, 1),
                "sustained_tflops": round(flops / (mean * 1e-3) / 1e12, 1),
                "how": f"torch._scaled_mm e4m3 x e4m3 -> bf16, {n}^3: best of 10 (burst), mean of {reps} back to "
                       f"back (sustained)"}
    except Exception as e:  # library without FP8 GEMM support: reported, not fatal
        return {"error": f"{type(e).__name__}: {e}"[:200]}


def setup_workload(pg, torch, dev, name):
    """Weights quantised per channel (or split into NestedFP planes) on the
    device, activations resident on the device and pinned on the host,
    outputs and zero-filled workspaces: everything a step reads or writes."""
    copies = weight_copies(name)
    layers = workload_layers(name, copies)
    weights = {}
    for L in layers:
        key = (L.shape_idx, L.copy, L.kind in ("nested16", "nested8"))
        if key in weights:
            continue
        w = torch.from_numpy(synthetic.weights(base_workload(name), L.shape_idx, copy=L.copy)).to(dev)
        weights[key] = pg.nestedfp_split(w) if key[2] else pg.fp8_quantize_rows(w)
        del w
    acts_host, acts, outs, qbufs = [], [], [], []
    for L in layers:
        x = synthetic.acts(base_workload(name), L.shape_idx, L.m_idx)
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
    return dict(name=name, copies=copies, layers=layers, weights=weights, acts_host=acts_host, acts=acts,
                outs=outs, qbufs=qbufs)


def _wkey(L):
    return (L.shape_idx, L.copy, L.kind != "fp8")


GROUP_MAX_M = 256   # the library's grouped weight-streaming kernel takes layers up to this many tokens


class StepRunner:
    """Enqueues one step of a workload on `stream` through the C ABI.

    Grouped form (FP8 workloads, per-token dynamic scales, the default): one
    pgf8_fp8_linear_dynamic_group call for every layer of the step.  The
    per-layer form (--per-layer, and every option that changes the layers'
    producers) chains one call per layer with PGF8_FLAG_OVERLAP_PREVIOUS.

    The bracketed step (for the roofline) runs the same launches with an
    event between consecutive launch groups: the quantisation and the
    grouped kernel on the M <= 128 layers, then the quantisation of the
    larger layers and their tiled launch on SM pairs
    (pgf8_fp8_linear_group); its intervals are scaled to the timed step."""

    def __init__(self, pg, torch, dev, wl, args, stream):
        self.pg, self.torch, self.dev, self.wl, self.args, self.stream = pg, torch, dev, wl, args, stream
        layers = wl["layers"]
        self.layers = layers
        plain = not args.per_layer and not args.chain and args.scaling == "dynamic" and not args.fused_quant
        self.grouped = plain and all(L.kind == "fp8" for L in layers)
        # NestedFP workloads: one pgf8_nestedfp_linear_group call per mode
        self.nested_grouped = plain and all(L.kind in ("nested16", "nested8") for L in layers)
        self.xflags = pg.FLAG_FUSED_QUANT if args.fused_quant else 0
        self.sk_ws = torch.zeros(max(16, max(pg.lib.pgf8_fp8_linear_workspace_size(L.M, L.N, L.K) for L in layers)),
                                 dtype=torch.uint8, device=dev)
        if self.grouped:
            ent = lambda i: (wl["acts"][i], *wl["weights"][_wkey(layers[i])], wl["outs"][i], wl["qbufs"][i])  # noqa: E731
            self.group = pg.LayerGroup([ent(i) for i in range(len(layers))])
            # the library's launches for a group: the quantisation and the
            # grouped kernel on the M <= 128 layers (32 per launch), then the
            # quantisation and the tiled launch on SM pairs over all the
            # larger layers (32 per launch)
            small = [i for i, L in enumerate(layers) if L.M <= 128]
            large = [i for i, L in enumerate(layers) if L.M > 128]
            self.classes = [small[j:j + 32] for j in range(0, len(small), 32)]
            self.large_chunks = [large[j:j + 32] for j in range(0, len(large), 32)]
            self.large = large
            self.sub = [pg.LayerGroup([ent(i) for i in idx]) for idx in self.classes]
        if self.nested_grouped:
            def nent(i):
                L = layers[i]
                hi, lo = wl["weights"][_wkey(L)]
                n16 = L.kind == "nested16"
                return (wl["acts"][i], hi, lo if n16 else None, wl["outs"][i], None if n16 else wl["qbufs"][i])
            self.ngroups, self.nsub, self.nlarge = [], [], []
            for kind in ("nested16", "nested8"):
                mode = pg.NESTED_FP16 if kind == "nested16" else pg.NESTED_FP8
                idx = [i for i, L in enumerate(layers) if L.kind == kind]
                if not idx:
                    continue
                self.ngroups.append(pg.NestedLayerGroup([nent(i) for i in idx], mode=mode))
                for lo_m, hi_m in ((0, 128), (128, GROUP_MAX_M)):
                    cls = [i for i in idx if lo_m < layers[i].M <= hi_m]
                    for j in range(0, len(cls), 32):
                        self.nsub.append((cls[j:j + 32], pg.NestedLayerGroup([nent(i) for i in cls[j:j + 32]],
                                                                             mode=mode)))
                self.nlarge += [i for i in idx if layers[i].M > GROUP_MAX_M]
        self.per_tensor = {}
        if not self.grouped and args.scaling != "dynamic":
            for i, L in enumerate(layers):
                if L.kind == "fp8":
                    self.per_tensor[i] = (pg.DelayedScaling(1024, device=dev) if args.scaling == "delayed"
                                          else pg.fp8_amax_accumulate(wl["acts"][i]))
            torch.cuda.synchronize()
        self.gammas = {}
        if args.chain:
            if any(L.kind != "fp8" for L in layers) or len(synthetic.WORKLOADS[wl["name"]].shapes) != 4:
                raise SystemExit("--chain needs a workload of QKV, O, gate+up, down FP8 layers")
            g = torch.Generator().manual_seed(7)
            for i, L in enumerate(layers):
                if L.shape_idx in (0, 2):
                    self.gammas[i] = (0.5 + torch.rand(L.K, generator=g)).to(dev)

    # -- launches -------------------------------------------------------------------------------------------------
    def launches_per_step(self):
        if self.grouped:
            return 2 * len(self.classes) + 2 * len(self.large_chunks)
        if self.nested_grouped:
            per = lambda i: 2 if self.layers[i].kind == "nested8" else 1  # noqa: E731
            return sum(per(idx[0]) for idx, _ in self.nsub) + sum(per(i) for i in self.nlarge)
        return sum(2 if L.kind in ("fp8", "nested8") else 1 for L in self.layers)

    def _quantise(self, i, L, flags):
        pg, wl, s = self.pg, self.wl, self.stream
        aq, sa = pg.dynamic_workspace_views(wl["qbufs"][i], L.M, L.K)
        if self.gammas and L.shape_idx in (0, 2):
            pg.fp8_norm_quantize(wl["acts"][i], self.gammas[i], None, 1e-6, aq, sa, flags=flags, stream=s)
        elif self.gammas and L.shape_idx == 3:
            pg.fp8_silu_mul_quantize(wl["outs"][i - 1], aq, sa, flags=flags, stream=s)
        elif i in self.per_tensor:
            if self.args.scaling == "delayed":
                self.per_tensor[i].step(wl["acts"][i], aq, sa, flags=flags, stream=s)
            else:
                pg.fp8_quantize_tensor(wl["acts"][i], self.per_tensor[i], aq, sa, flags=flags, stream=s)
        else:
            pg.fp8_quantize_rows(wl["acts"][i], aq, sa, stream=s)
        return aq, sa

    def step(self):
        """One step as a user runs it (no events)."""
        pg, wl, s = self.pg, self.wl, self.stream
        if self.grouped:
            self.group.run(flags=pg.FLAG_OVERLAP_PREVIOUS, stream=s)
            return
        if self.nested_grouped:
            for grp in self.ngroups:
                grp.run(flags=pg.FLAG_OVERLAP_PREVIOUS, stream=s)
            return
        ov = pg.FLAG_OVERLAP_PREVIOUS
        for i, L in enumerate(self.layers):
            W = wl["weights"][_wkey(L)]
            if L.kind == "fp8":
                if not self.gammas and not self.per_tensor:
                    pg.fp8_linear_dynamic(wl["acts"][i], W[0], W[1], y=wl["outs"][i], workspace=wl["qbufs"][i],
                                          flags=ov | self.xflags, stream=s)
                    continue
                if self.gammas and L.shape_idx == 1:   # O: dynamic pair, overlapped
                    pg.fp8_linear_dynamic(wl["acts"][i], W[0], W[1], y=wl["outs"][i], workspace=wl["qbufs"][i],
                                          flags=ov, stream=s)
                    continue
                aq, sa = self._quantise(i, L, ov)
                pg.fp8_linear(aq, sa, W[0], W[1], y=wl["outs"][i], workspace=self.sk_ws, flags=ov, stream=s)
            else:
                mode = pg.NESTED_FP16 if L.kind == "nested16" else pg.NESTED_FP8
                pg.nestedfp_linear(wl["acts"][i], W[0], W[1] if mode == pg.NESTED_FP16 else None, mode=mode,
                                   y=wl["outs"][i], workspace=wl["qbufs"][i], flags=ov | self.xflags, stream=s)

    def bracketed_step(self, marks):
        """The same kernels with an event recorded before every launch group
        and one at the end: marks.append((segment, event))."""
        pg, wl, s, torch = self.pg, self.wl, self.stream, self.torch

        def mark(seg):
            e = torch.cuda.Event(enable_timing=True, external=True)
            e.record(s)
            marks.append((seg, e))

        if self.grouped:
            for idx, sub in zip(self.classes, self.sub):
                mark(("group", tuple(idx)))
                sub.run(stream=s)
            for chunk in self.large_chunks:
                mark(("quant", tuple(chunk)))
                ops = []
                for i in chunk:
                    L = self.layers[i]
                    W = wl["weights"][_wkey(L)]
                    aq, sa = self._quantise(i, L, 0)
                    ops.append((aq, sa, W[0], W[1], wl["outs"][i]))
                mark(("gemm", tuple(chunk)))
                pg.fp8_linear_group(ops, stream=s)
        elif self.nested_grouped:
            for idx, sub in self.nsub:
                mark(("group", tuple(idx)))
                sub.run(stream=s)
            for i in self.nlarge:
                L = self.layers[i]
                W = wl["weights"][_wkey(L)]
                mode = pg.NESTED_FP16 if L.kind == "nested16" else pg.NESTED_FP8
                mark(("gemm", (i,)))
                pg.nestedfp_linear(wl["acts"][i], W[0], W[1] if mode == pg.NESTED_FP16 else None, mode=mode,
                                   y=wl["outs"][i], workspace=wl["qbufs"][i], stream=s)
        else:
            for i, L in enumerate(self.layers):
                W = wl["weights"][_wkey(L)]
                if L.kind == "fp8":
                    mark(("quant", (i,)))
                    aq, sa = self._quantise(i, L, 0)
                    mark(("gemm", (i,)))
                    pg.fp8_linear(aq, sa, W[0], W[1], y=wl["outs"][i], workspace=self.sk_ws, stream=s)
                else:
                    mode = pg.NESTED_FP16 if L.kind == "nested16" else pg.NESTED_FP8
                    mark(("gemm", (i,)))
                    pg.nestedfp_linear(wl["acts"][i], W[0], W[1] if mode == pg.NESTED_FP16 else None, mode=mode,
                                       y=wl["outs"][i], workspace=wl["qbufs"][i], flags=self.xflags, stream=s)
        mark(("end", ()))


def quant_bytes(L):
    xb = 2 if L.kind.startswith("nested") else 4
    return L.M * L.K * (xb + 1) + 4 * L.M


def analyse_segments(layers, marks, ms_step, peaks, fp8_peak, long_region=True):
    """Per-segment durations of the bracketed step, scaled so that they sum
    to the timed step (a kernel's share of the step times the step), the
    dominant kernel's roofline and the regime checks of the layer's targets,
    over the segments whose layers all fall in the regime: decode (M <= 16)
    >= 80 % of HBM; weight streaming (M <= 128: the grouped kernel; the
    M = 256 layers join the tiled launch, at the FP8 ridge) >= 75 % of HBM;
    prefill (M >= 512) >= 60 % of the FP8 tensor peak.

    marks: (segment, event, ms since the previous mark); segment k runs
    from mark k to mark k + 1.  Tensor peaks: the measured bf16 figure
    (x 2 for E4M3 MMAs) sustained when the timed region ran long or under
    the power cap (long_region), else the burst figure."""
    segs = []
    for (seg, _, _), (_, _, dt) in zip(marks[:-1], marks[1:]):
        kind, idx = seg
        segs.append({"kind": kind, "layers": list(idx), "ms": dt})
    total = sum(sg["ms"] for sg in segs)
    scale = ms_step / total if total > 0 else 1.0
    hbm = float(peaks["hbm_gbs"])
    sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    if not long_region:
        sustained = float(peaks["bf16_tflops"])   # burst: a short timed region, no power cap seen
    fp8_peak_tf = 2.0 * sustained
    out = []
    cls_time, cls_bytes, cls_flops = {}, {}, {}
    for sg in segs:
        Ls = [layers[i] for i in sg["layers"]]
        t_in = sg["ms"] * scale
        if sg["kind"] == "quant":
            b = sum(quant_bytes(L) for L in Ls)
            f = 0.0
        else:
            b = sum(L.gemm_bytes for L in Ls)
            f = sum(L.flops for L in Ls)
        wb = sum(L.weight_bytes for L in Ls) if sg["kind"] != "quant" else 0
        cls = sg["kind"]
        cls_time[cls] = cls_time.get(cls, 0.0) + t_in
        cls_bytes[cls] = cls_bytes.get(cls, 0.0) + b
        cls_flops[cls] = cls_flops.get(cls, 0.0) + f
        out.append({"kind": sg["kind"], "M": sorted({L.M for L in Ls}), "shapes": len(Ls),
                    "us_bracketed": round(sg["ms"] * 1e3, 2), "us_in_step": round(t_in * 1e3, 2),
                    "gbs": round(b / (t_in * 1e-3) / 1e9, 1) if t_in > 0 else None,
                    "weight_gbs": round(wb / (t_in * 1e-3) / 1e9, 1) if (t_in > 0 and wb) else None,
                    "tflops": round(f / (t_in * 1e-3) / 1e12, 1) if (t_in > 0 and f) else None})
    def peak_of(L):   # dense tensor peak of the layer's MMA kind (TFLOP/s)
        return sustained if L.kind == "nested16" else fp8_peak_tf

    dom = max(cls_time, key=cls_time.get)
    t = cls_time[dom] * 1e-3
    if dom == "gemm" and any(layers[i].M > 256 for sg in segs if sg["kind"] == "gemm" for i in sg["layers"]):
        achieved = cls_flops[dom] / t / 1e12
        dom_layers = [layers[i] for sg in segs if sg["kind"] == dom for i in sg["layers"]]
        ideal_s = sum(L.flops / (peak_of(L) * 1e12) for L in dom_layers)
        peak_eff = cls_flops[dom] / ideal_s / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak_eff, 1),
                "unit": "TFLOP/s", "frac": round(ideal_s / t, 4),
                "peak_source": ("measured bf16 sustained (MEASURED_PEAKS.json) x 2 for E4M3 MMAs (the FP8/bf16 "
                                "nominal ratio), x 1 for FP16 MMAs; kernels timed inside a long power-capped "
                                "region") if long_region else
                               ("measured bf16 burst (MEASURED_PEAKS.json) x 2 for E4M3 MMAs, x 1 for FP16 MMAs; "
                                "a short timed region without the power cap")}
        if fp8_peak and "sustained_tflops" in fp8_peak:
            roof["frac_of_scaled_mm_fp8_sustained"] = round(achieved / fp8_peak["sustained_tflops"], 4)
            roof["frac_of_scaled_mm_fp8_burst"] = round(achieved / fp8_peak["burst_tflops"], 4)
        roof["kernel"] = "pgf8::gemm_pair_kernel / gemm_persistent_kernel (tiled GEMMs of the M > 128 layers)"
    else:
        achieved = cls_bytes[dom] / t / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4),
                "peak_source": "measured HBM copy bandwidth (MEASURED_PEAKS.json)"}
        roof["kernel"] = ("pgf8::gemm_group_kernel (with its quantisation launch)" if dom == "group"
                          else "pgf8::gemm_kernel")
    roof["dominant_class"] = dom
    roof["kernel_ms_per_step"] = round(cls_time[dom], 5)
    roof["share_of_step"] = round(cls_time[dom] / ms_step, 4)
    roof["bracketed_over_timed_step"] = round(total / ms_step, 4)
    roof["algorithmic_per_step"] = (f"{cls_flops[dom]:.4e} flop" if roof["bound"] == "tensor"
                                    else f"{cls_bytes[dom]:.4e} B")

    def regime(pred, what, kind=None):
        t_s = wbytes = fl = ideal = 0.0
        for sg in segs:
            Ls = [layers[i] for i in sg["layers"]]
            if Ls and all(pred(L.M) and (kind is None or L.kind == kind) for L in Ls):
                t_s += sg["ms"] * scale * 1e-3
                if sg["kind"] != "quant":
                    wbytes += sum(L.weight_bytes for L in Ls)
                    fl += sum(L.flops for L in Ls)
                    ideal += sum(L.flops / (peak_of(L) * 1e12) for L in Ls)
        if t_s == 0:
            return None
        if what == "hbm":
            gbs = wbytes / t_s / 1e9
            return {"weight_gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}
        tf = fl / t_s / 1e12
        r = {"tflops": round(tf, 1), "frac_fp8_peak": round(ideal / t_s, 4)}
        if fp8_peak and "sustained_tflops" in fp8_peak:
            r["frac_scaled_mm_fp8_sustained"] = round(tf / fp8_peak["sustained_tflops"], 4)
        return r

    regimes = {}
    for key, pred, what, target in (("decode_m_le_16", lambda m: m <= 16, "hbm", 0.80),
                                    ("weight_streaming_m_le_128", lambda m: m <= 128, "hbm", 0.75),
                                    ("prefill_m_ge_512", lambda m: m >= 512, "tensor", 0.60)):
        r = regime(pred, what)
        if r is not None:
            frac = r["frac_hbm"] if what == "hbm" else r["frac_fp8_peak"]
            r["target"] = target
            r["pass"] = bool(frac >= target)
            regimes[key] = r
    # NestedFP: the decode regime of each mode on its own
    for kind, tag in (("nested16", "fp16_mode"), ("nested8", "fp8_mode")):
        if any(L.kind == kind for L in layers):
            r = regime(lambda m: m <= 16, "hbm", kind)
            if r is not None:
                r["target"] = 0.80
                r["pass"] = bool(r["frac_hbm"] >= 0.80)
                regimes["decode_m_le_16_" + tag] = r
    return roof, regimes, out


def time_workload(pg, torch, dev, wl, args, steps, warmup, world, peaks, fp8_peak, clocks=False):
    """Graph of R steps replayed (steps / R) times between barriers and
    synchronizes, CUDA events on the launching stream, max over ranks; then
    one bracketed step for the per-kernel shares."""
    stream = torch.cuda.Stream(device=dev)
    runner = StepRunner(pg, torch, dev, wl, args, stream)
    layers = wl["layers"]
    R = max(1, min(10, steps))
    while steps % R:
        R -= 1
    with torch.cuda.stream(stream):
        runner.step()                      # first-call set-up outside capture
        runner.bracketed_step([])
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(R):
            runner.step()
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-warmup // R))):
            graph.replay()
    torch.cuda.synchronize()
    if pg.device_status(stream) != pg.OK:
        raise RuntimeError("device error word raised during warm-up")

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    sampler = ClockSampler(dev.index or 0) if clocks else None
    if sampler:
        sampler.start()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps // R):
            graph.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = sampler.stop() if sampler else None
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, dev)
    st = pg.device_status(stream)
    if st != pg.OK:
        raise RuntimeError(f"device error word raised in the timed region: {st}")
    ms_step = ms_total / steps

    # bracketed steps (outside the timed region), replayed from a CUDA graph
    # like the timed steps, so that no host launch gap sits between two
    # events: first as many replays back to back as the timed region had
    # steps (the GPU reaches the same power state, under the power cap the
    # same clocks), then 3 measured replays, the middle one by total time
    runs = []
    bracket_mode = "graph"
    try:
        marks_g = []
        bgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(bgraph, stream=stream):
            runner.bracketed_step(marks_g)
        with torch.cuda.stream(stream):
            for _ in range(steps):
                bgraph.replay()
        stream.synchronize()
        for _ in range(3):
            with torch.cuda.stream(stream):
                bgraph.replay()
            stream.synchronize()
            runs.append([(seg, ev, seg_ev.elapsed_time(ev) if k else 0.0)
                         for k, ((seg, ev), (_, seg_ev)) in enumerate(zip(marks_g, [marks_g[0]] + marks_g[:-1]))])
        del bgraph
    except RuntimeError:
        # (events recorded inside a capture not supported): eager launches
        torch.cuda.synchronize()
        bracket_mode = "eager"
        runs = []
        for _ in range(3):
            marks = []
            with torch.cuda.stream(stream):
                runner.bracketed_step(marks)
            stream.synchronize()
            runs.append([(seg, ev, prev.elapsed_time(ev) if k else 0.0)
                         for k, ((seg, ev), (_, prev)) in enumerate(zip(marks, [marks[0]] + marks[:-1]))])
    # keep the middle run by total bracketed time
    totals = [sum(d for (_, _, d) in r) for r in runs]
    marks = runs[sorted(range(3), key=lambda k: totals[k])[1]]
    long_region = ms_total >= 200.0 or bool(clk and "sw_power_cap" in clk.get("reasons", []))
    roof, regimes, segments = analyse_segments(layers, marks, ms_step, peaks, fp8_peak, long_region)
    roof["bracketing"] = bracket_mode
    del graph
    wbytes = sum(L.weight_bytes for L in layers)
    flops = sum(L.flops for L in layers)
    return dict(runner=runner, ms_step=ms_step, R=R, wbytes=wbytes, flops=flops, roof=roof, regimes=regimes,
                segments=segments, clocks=clk, launches=runner.launches_per_step())


def run_ours(args, rank, world, local_rank):
    import torch
    import precision_gemm_fp8_b200 as pg

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = _load_peaks()
    name = args.workload
    fp8_peak = measure_fp8_peak(torch, dev) if not args.no_fp8_peak else None
    wl = setup_workload(pg, torch, dev, name)
    layers = wl["layers"]
    K, W = args.steps, args.warmup
    res = time_workload(pg, torch, dev, wl, args, K, W, world, peaks, fp8_peak, clocks=True)
    ms_step = res["ms_step"]
    wbytes, flops = res["wbytes"], res["flops"]
    gbs = job_throughput(wbytes / 1e9, world, ms_step * 1e-3)        # whole job, all ranks
    tflops = job_throughput(flops / 1e12, world, ms_step * 1e-3)
    memory_bound = name in ("decode7b", "nested7b_decode", "small")
    roof = res["roof"]
    roof["traffic"], roof["traffic_note"] = profiled_traffic(name)
    if fp8_peak is not None:
        roof["fp8_scaled_mm_measured"] = fp8_peak
    roof["peak_file"] = peak_src

    # ---- e2e through the public entry point, host buffers, copies inside the timed region
    e2e = run_e2e(pg, torch, dev, wl, args, world, wbytes, flops, memory_bound)

    grouped = res["runner"].grouped
    nested_grouped = res["runner"].nested_grouped
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
                         % (wl["copies"], wbytes / 1e6),
                   "step": ("one pgf8_fp8_linear_dynamic_group call: the M <= 128 layers quantised by one launch and "
                            "streamed by one grouped kernel, each larger layer quantised and multiplied by its own "
                            "kernels" if grouped else
                            "one pgf8_nestedfp_linear_group call per mode: its M <= 128 layers streamed by one "
                            "grouped kernel, each larger layer by the tiled kernels" if nested_grouped else
                            "one call per layer, chained with PGF8_FLAG_OVERLAP_PREVIOUS"),
                   "timing": "CUDA graph of the C-ABI calls, R=%d steps per replay, replayed K/R times" % res["R"],
                   "quantisation": ("inside the skinny GEMM where each CTA's activation slice fits its registers"
                                    if args.fused_quant else "per token, dynamic, own kernel before the GEMM"),
                   "chain": ("decoder layer: RMSNorm+quantise -> QKV; quantise -> O; RMSNorm+quantise -> "
                             "gate+up; SiLU gate+quantise of the gate+up output -> down") if args.chain else None,
                   "activation_scaling": {"dynamic": "per token, dynamic",
                                          "delayed": "per tensor, delayed (amax history of 1024 per layer)",
                                          "static": "per tensor, MINMAX-calibrated amax"}[args.scaling]},
        "secondary": {"tflops": round(tflops, 3), "weight_gbs": round(gbs, 1), "regimes": res["regimes"]},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": int(res["launches"] * K),
        "clocks": res["clocks"],
        "segments": res["segments"],
    }
    del wl, res
    torch.cuda.empty_cache()

    # ---- the other configurations, each timed as its own step in this run
    if not args.no_secondary and name == "llama70b":
        for sec in ("decode7b", "prefill7b", "nested7b", "nested7b_decode"):
            wl2 = setup_workload(pg, torch, dev, sec)
            steps2 = {"decode7b": 400, "prefill7b": 60, "nested7b": 60, "nested7b_decode": 200}[sec]
            r2 = time_workload(pg, torch, dev, wl2, args, steps2, 10, world, peaks, fp8_peak)
            r2["roof"]["traffic"], r2["roof"]["traffic_note"] = profiled_traffic(sec)
            mb = sec in ("decode7b", "nested7b_decode")
            v = (r2["wbytes"] / 1e9 if mb else r2["flops"] / 1e12) / (r2["ms_step"] * 1e-3) * world
            result["secondary"][sec] = {
                "value": round(v, 2), "unit": "GB/s" if mb else "TFLOP/s", "ms_per_step": round(r2["ms_step"], 5),
                "steps": steps2, "grouped": r2["runner"].grouped or r2["runner"].nested_grouped,
                "roofline": r2["roof"], "regimes": r2["regimes"],
                "segments": r2["segments"]}
            if sec == "decode7b" and "decode_m_le_16" in r2["regimes"]:
                # the decode regime as its own step (the 70B step streams its
                # M <= 16 layers together with the M <= 128 ones)
                result["secondary"]["regimes"]["decode_m_le_16"] = dict(r2["regimes"]["decode_m_le_16"],
                                                                        measured_on="decode7b step")
            del wl2, r2
            torch.cuda.empty_cache()
    return result


def run_e2e(pg, torch, dev, wl, args, world, wbytes, flops, memory_bound):
    """The metric end to end through the public API with host buffers: every
    step copies all of its activations from a pinned host buffer to the
    device, runs the step (one pgf8_fp8_linear_dynamic_group call for the FP8
    workloads, one call per layer otherwise) and copies all of its outputs
    back to a pinned host buffer; the copies are inside the timed region.

    Steps are pipelined as a server runs them: two device buffer sets, the
    host-to-device copies on one stream, the kernels on a second and the
    device-to-host copies on a third, so step k's outputs go back to the host
    while step k+1's inputs come in and step k+1 computes (PCIe carries both
    directions at once).  Events order the buffers: a step's inputs are not
    overwritten before the step that reads them has computed, its outputs not
    before they have been copied out."""
    layers, acts_host, outs = wl["layers"], wl["acts_host"], wl["outs"]
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))

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
    ws = [torch.zeros_like(q) for q in wl["qbufs"]]
    bufs = []
    for _ in range(2):
        x_dev, x_views = packed(acts_host, dev)
        x_dev.copy_(x_host)      # calibrated per-tensor scales (--scaling static) read the inputs at set-up
        y_dev, y_views = packed(outs, dev)
        y_host, _ = packed(outs, "cpu")
        torch.cuda.synchronize()
        runner = StepRunner(pg, torch, dev, dict(wl, acts=x_views, outs=y_views, qbufs=ws), args, s_comp)
        ev = {k: torch.cuda.Event() for k in ("in", "comp", "out")}
        bufs.append(dict(x_dev=x_dev, y_dev=y_dev, y_host=y_host, runner=runner, ev=ev, used=False))

    def step(k):
        b = bufs[k % 2]
        if b["used"]:
            s_in.wait_event(b["ev"]["comp"])       # the previous step on these buffers has read its inputs
        with torch.cuda.stream(s_in):
            b["x_dev"].copy_(x_host, non_blocking=True)
            b["ev"]["in"].record(s_in)
        s_comp.wait_event(b["ev"]["in"])
        if b["used"]:
            s_comp.wait_event(b["ev"]["out"])      # ... and its outputs have been copied out
        with torch.cuda.stream(s_comp):
            b["runner"].step()
            b["ev"]["comp"].record(s_comp)
        s_out.wait_event(b["ev"]["comp"])
        with torch.cuda.stream(s_out):
            b["y_host"].copy_(b["y_dev"], non_blocking=True)
            b["ev"]["out"].record(s_out)
        b["used"] = True

    steps = max(3, min(args.steps, 100))
    for k in range(4):
        step(k)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for k in range(steps):
        step(k)
    t1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    v = job_throughput(wbytes / 1e9 if memory_bound else flops / 1e12, world, ms * 1e-3)
    return {"value": round(v, 2), "unit": "GB/s" if memory_bound else "TFLOP/s",
            "h2d_bytes_per_step": int(x_host.numel()), "d2h_bytes_per_step": int(bufs[0]["y_host"].numel()),
            "steps": steps, "ms_per_step": round(ms, 5),
            "pipeline": "two device buffer sets; H2D, kernels and D2H on three streams ordered by events",
            "entry_point": ("pgf8_fp8_linear_dynamic_group" if bufs[0]["runner"].grouped else
                            "pgf8_nestedfp_linear_group" if bufs[0]["runner"].nested_grouped else
                            "one C-ABI call per layer (pgf8_fp8_linear_dynamic / pgf8_nestedfp_linear / the "
                            "scaling and producer variants + pgf8_fp8_linear)")}


# ----------------------------------------------------------------------------- CPU oracle
ORACLE_SAMPLE = {  # per layer: first `rows` tokens x first `cols` output channels
    "small": (16, 512), "decode7b": (8, 256), "prefill7b": (16, 48), "nested7b": (16, 96), "nested7b_decode": (16, 96), "llama70b": (16, 64),
}


def oracle_inputs(name, rows=None, cols=None):
    """Inputs of the bounded oracle sample of one step of the workload (not
    timed): for every layer, its first `rows` tokens and the weights of its
    first `cols` output channels, quantised / split as the layer stores them
    (the weights' offline preparation is not part of the step)."""
    import oracle

    r0, c0 = ORACLE_SAMPLE[name]
    rows, cols = rows or r0, cols or c0
    items = []
    for L in workload_layers(name, weight_copies(name)):
        m = min(rows, L.M)
        x = synthetic.acts(base_workload(name), L.shape_idx, L.m_idx, M=m)
        nc = min(cols, L.N)
        w = synthetic.weights(base_workload(name), L.shape_idx, copy=L.copy, n_override=nc)
        prep = oracle.quantize_rows(w) if L.kind == "fp8" else oracle.nestedfp_split(w)
        items.append((L, x, prep))
    desc = (f"all {len(items)} layers of one step, each on its first {rows} tokens (quantised over the full K) x "
            f"first {cols} output channels; value = work computed / seconds (no extrapolation)")
    return items, desc


def oracle_run(items, threads, pool=None):
    """Time the CPU oracle, as it stands, on prepared sample inputs: the
    per-token quantisation and the binary64 contraction of every layer, the
    output channels split over `threads` host threads (the oracle is a C
    library called through ctypes, which releases the interpreter lock, so
    nothing of its arithmetic changes).  Returns (seconds, flops, weight bytes)."""
    import oracle

    total = flops = wbytes = 0.0
    for L, x, prep in items:
        nc = prep[0].shape[0]
        parts = [p for p in np.array_split(np.arange(nc), threads) if p.size]
        t0 = time.perf_counter()
        if L.kind == "fp8":
            wq, sw = prep
            aq, sa = oracle.quantize_rows(x)
            fn = lambda p: oracle.fp8_linear(aq, sa, wq[p[0]:p[-1] + 1], sw[p[0]:p[-1] + 1])  # noqa: E731
        elif L.kind == "nested16":
            hi, lo = prep
            fn = lambda p: oracle.nestedfp_linear_fp16(x, hi[p[0]:p[-1] + 1], lo[p[0]:p[-1] + 1])  # noqa: E731
        else:
            hi = prep[0]
            fn = lambda p: oracle.nestedfp_linear_fp8(x, hi[p[0]:p[-1] + 1])  # noqa: E731
        if pool is not None and len(parts) > 1:
            list(pool.map(fn, parts))
        else:
            fn(np.arange(nc))
        total += time.perf_counter() - t0
        flops += 2.0 * x.shape[0] * nc * L.K
        wbytes += nc * L.K * (2 if L.kind == "nested16" else 1)
    return total, flops, wbytes


def cpu_baseline_entry(name, unit):
    from concurrent.futures import ThreadPoolExecutor

    threads = os.cpu_count() or 1
    items, desc = oracle_inputs(name)
    val = (lambda s, f, b: (b / s / 1e9) if unit == "GB/s" else (f / s / 1e12))
    with ThreadPoolExecutor(threads) as pool:
        sn, fn_, bn = oracle_run(items, threads, pool)
        s1, f1, b1 = oracle_run(items, 1)
        out = {"value": val(sn, fn_, bn), "unit": unit, "cores": threads, "kind": "oracle", "sample": desc,
               "sample_seconds": round(sn, 3),
               "single_thread": {"value": val(s1, f1, b1), "cores": 1, "sample_seconds": round(s1, 3)},
               "host_cpus": os.cpu_count()}
        if name in ("llama70b", "decode7b"):
            # the decode7b step at M = 1 with every output channel of every layer
            full, _ = oracle_inputs("decode7b", rows=1, cols=1 << 30)
            full = [it for it in full if it[0].M == 1]
            t, f, b = oracle_run(full, threads, pool)
            out["decode7b_m1_full"] = {"weight_gbs": round(b / t / 1e9, 5), "tflops": f / t / 1e12,
                                       "seconds": round(t, 3), "cores": threads,
                                       "sample": "decode7b at M = 1: all four layers, every output channel"}
    return out


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores; each
    step is one bounded sample of the workload (every layer on its first
    tokens x first output channels), sized so the whole --steps/--warmup run
    takes about two minutes.  value = work computed / time, ms_per_step = the
    sample's own time."""
    from concurrent.futures import ThreadPoolExecutor

    name = args.workload
    memory_bound = name in ("decode7b", "nested7b_decode", "small")
    threads = os.cpu_count() or 1
    r0, c0 = ORACLE_SAMPLE[name]
    with ThreadPoolExecutor(threads) as pool:
        probe, _ = oracle_inputs(name, rows=r0, cols=max(1, c0 // 8))
        s, _, _ = oracle_run(probe, threads, pool)
        budget = max(0.05, 100.0 / (args.warmup + args.steps))
        cols = int(max(1, min(c0 * 8, max(1, c0 // 8) * budget / max(s, 1e-6))))
        items, desc = oracle_inputs(name, rows=r0, cols=cols)
        times, fl, wb = [], 0.0, 0.0
        for i in range(args.warmup + args.steps):
            s, f, b = oracle_run(items, threads, pool)
            if i >= args.warmup:
                times.append(s)
                fl, wb = f, b
    ms = 1e3 * sum(times) / len(times)
    v = (wb / (ms * 1e-3) / 1e9) if memory_bound else (fl / (ms * 1e-3) / 1e12)
    unit = "GB/s" if memory_bound else "TFLOP/s"
    return {
        "metric": METRIC, "value": v, "unit": unit, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{name}: {WORKLOAD_TEXT[name]}"},
        "cpu_baseline": {"kind": "oracle", "cores": threads, "sample": desc, "value": v, "unit": unit},
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
    elif kind == "group":
        # the layer as a grouped call of one (M <= 256: the grouped weight-streaming kernel)
        wq, sw = pg.fp8_quantize_rows(w)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(pg.fp8_linear_dynamic_workspace_size(M, N, K), dtype=torch.uint8, device=dev)
        grp = pg.LayerGroup([(x, wq, sw, y, ws)])
        fn = grp.run
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(synthetic.WORKLOADS) + sorted(BASE_WORKLOAD), default="llama70b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="llama70b: skip timing decode7b, prefill7b and nested7b as secondary steps")
    ap.add_argument("--no-fp8-peak", action="store_true", help="skip the torch._scaled_mm FP8 reference figure")
    ap.add_argument("--per-layer", action="store_true",
                    help="one C-ABI call per layer, chained (the form a dependent layer sequence runs in) instead "
                         "of one grouped call per step")
    ap.add_argument("--scaling", choices=["dynamic", "delayed", "static"], default="dynamic",
                    help="activation scales of the FP8 layers: per-token dynamic (default), per-tensor delayed "
                         "(amax history of 1024) or per-tensor static (MINMAX-calibrated)")
    ap.add_argument("--chain", action="store_true",
                    help="feed each GEMM from its decoder-layer producer: RMSNorm fused with the quantisation ahead "
                         "of QKV and gate+up, the SiLU gate of the gate+up output ahead of down")
    ap.add_argument("--fused-quant", action="store_true",
                    help="quantise dynamic activations inside the skinny GEMM where its kernel allows it")
    ap.add_argument("--single", default=None, help="kind,M,K,N: time (or profile) one layer eagerly; kind = fp8 (pre-quantised "
                         "activations), dyn (dynamic), group (a grouped call of one), nested16, nested8")
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
                res["cpu_baseline"] = cpu_baseline_entry(args.workload, res["unit"])
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
