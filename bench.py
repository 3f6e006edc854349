#!/usr/bin/env python
"""Benchmark of the weight-quantized matmul hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A *step* is one pass over every matmul of the workload (default: the Llama-7B-shaped
W4A16 decode GEMVs, M in {1,4,16} x (N,K) in {(4096,4096),(11008,4096),(4096,11008)}),
each on its own copy of the packed weights: every case rotates through enough copies
that its copies together exceed 4x the 126 MB L2, so each launch streams its weights
from HBM.  Weights are quantized once on the GPU (offline step, untimed).

Timing: CUDA graphs of whole steps, replayed on one stream between CUDA events, after W
warm-up steps, with a barrier + torch.cuda.synchronize() on both sides; the max over ranks
is reported.  ``value`` = algorithmic bytes of all ranks / time (GB/s).  ``e2e`` repeats
the measurement through the same C-ABI calls with pinned HOST activations and outputs:
every step copies A host->device and C device->host inside the timed region.

Algorithmic bytes per launch: packed weights N*K*b/8 + scales (+ zeros) N*G*2 (each) +
activations M*K*2 (fp16/bf16; the INT8 paths quantize them per token inside the step) +
output M*N*2.

The default run also times, in the same process and the same way, the prefill GEMMs
("gemm": TFLOP/s against the measured bf16 tensor peak, burst and sustained), the W4A8
workload and the BitNet-3B ternary sweep, each with its per-case breakdown.

``--impl reference`` times the CPU oracle (plain C, float64) on a bounded sample of the
same workload on the host cores; it is a deliberately slow baseline, not a target.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

import wq_synth

ROOT = os.path.dirname(os.path.abspath(__file__))
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ------------------------------------------------------------------ workload arithmetic
def alg_bytes(c: wq_synth.Case) -> int:
    """Bytes the method must move for one matmul: packed weights, scales (+ zeros), the
    activations once and the output once.  The INT8 paths start from fp16 activations (the
    per-token quantization is part of the step), so they too read M*K*2 bytes of A; the
    INT8 copy of A and its scales are intermediate values, not counted."""
    bits = wq_synth.QUANT_BITS[c.quant]
    w = c.N * c.K * bits // 8
    if c.quant in ("tern2", "int1"):
        w += 4  # one binary32 scale
    else:
        G = c.K // c.group_size
        w += c.N * G * 2 * (2 if c.quant == "asym4" else 1)
    a = c.M * c.K * 2
    return w + a + c.M * c.N * 2


def flops(c: wq_synth.Case) -> int:
    return 2 * c.M * c.N * c.K


def launches_per_call(c: wq_synth.Case, fused: bool = True) -> int:
    """Kernels one step launches for the case: the matmul, plus the per-token activation
    quantization on the INT8 / FP8 paths, which for small activations (M <= 16, M*K <= 16384)
    runs inside the matmul kernel (w4a8_gemm_fused, w8a8_fp8_gemm_fused) and otherwise as a
    kernel of its own."""
    if c.mode not in ("a8", "f8"):
        return 1
    return 1 if (fused and c.M <= 16 and c.M * c.K <= 16384) else 2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS, "source": "fallback"}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "gemv_wq_quantize_b200", "csrc", "*"))):
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the workload's dominant kernel, from the committed ncu summary
    (profiles/<kernel>_<workload>.md), if it was taken of the current kernel sources."""
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"*_{workload}.md"))):
        fields = {}
        for line in open(path):
            if ":" in line and not line.startswith((" ", "#", "|")):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
        if fields.get("dominant") == "yes" and fields.get("source_sha") == kernel_source_hash():
            try:
                return float(fields["dram_bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(pynvml, device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    @staticmethod
    def _handle(nv, device):
        props = torch.cuda.get_device_properties(device)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                pass
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            dev = getattr(props, "pci_device_id", 0)
            try:
                return nv.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0")
            except Exception:
                pass
        return nv.nvmlDeviceGetHandleByIndex(0)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                break
            time.sleep(0.002)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nv:
            self.t.join()

    def report(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ our arm
def quant_config(c: wq_synth.Case):
    import gemv_wq_quantize_b200 as wq
    if c.quant == "tern2":
        return wq.QuantConfig(bits=2)
    if c.quant == "int1":
        return wq.QuantConfig(bits=1)
    if c.quant == "e2m1":
        return wq.QuantConfig(bits=4, group_size=c.group_size, format=wq.FMT_E2M1)
    if c.quant == "e4m3":
        return wq.QuantConfig(bits=8, group_size=c.group_size, format=wq.FMT_E4M3)
    return wq.QuantConfig(bits=4, group_size=c.group_size, symmetric=(c.quant == "sym4"))


class Prepared:
    """Quantized weight copies, activations and outputs of one case on the device."""

    def __init__(self, c: wq_synth.Case, device, seed_base: int = 0, copies: int = 0, fused: bool = True,
                 native: bool = False):
        import dataclasses
        import gemv_wq_quantize_b200 as wq
        self.c = c
        self.fused = fused
        self.qc = quant_config(c)
        W = wq_synth.weights(c.N, c.K, seed=seed_base).to(device)
        Wq, s, z = wq.quantize_pack(W, self.qc)
        del W
        if native:  # the kernel-native copy of the same weights
            Wq = wq.repack(Wq, c.N, c.K, self.qc)
            self.qc = dataclasses.replace(self.qc, layout=wq.LAYOUT_NATIVE)
        self.bytes = alg_bytes(c)
        copies = copies or max(2, math.ceil(4 * L2_BYTES / self.bytes))
        self.weights = [(Wq, s, z)] + [(Wq.clone(), s.clone(), None if z is None else z.clone())
                                        for _ in range(copies - 1)]
        A = wq_synth.activations(c.M, c.K, seed=seed_base + 1, dtype=c.a_dtype, outlier_frac=c.outlier_frac)
        self.A = A.to(device)
        self.A_host = A.pin_memory()
        if c.mode == "a8":
            self.Aq, self.a_scale = wq.act_quant_int8(self.A)
        elif c.mode == "f8":
            self.Aq, self.a_scale = wq.act_quant_fp8(self.A)
        self.C = torch.empty(c.M, c.N, dtype=torch.float16 if c.mode in ("a8", "f8") else c.a_dtype, device=device)
        self.C_host = torch.empty(self.C.shape, dtype=self.C.dtype).pin_memory()
        self.ws = wq.make_workspace(wq.workspace_size(c.M, c.N, c.K, self.qc), device)
        self.i = 0

    def launch(self, e2e: bool = False, slot: int = 0):
        import gemv_wq_quantize_b200 as wq
        Wq, s, z = self.weights[self.i % len(self.weights)]
        self.i += 1
        c = self.c
        A, C = (self.A_slots[slot], self.C_slots[slot]) if e2e else (self.A, self.C)
        if c.mode == "a16":
            wq.w4a16_gemm(A, Wq, s, z, c.N, c.K, self.qc, out=C, workspace=self.ws)
        elif c.mode == "f8" and self.fused:
            # FP8 x FP8: the step quantizes the fp16 activations per token (inside the matmul for
            # small activations), then multiplies
            wq.w8a8_fp8_gemm_fused(A, Wq, s, c.N, c.K, self.qc, out=C, out_q=self.Aq, out_scale=self.a_scale,
                                   workspace=self.ws)
        elif c.mode == "f8":
            wq.act_quant_fp8(A, out_q=self.Aq, out_scale=self.a_scale)
            wq.w8a8_fp8_gemm(self.Aq, self.a_scale, Wq, s, c.N, c.K, self.qc, out=C, workspace=self.ws)
        elif self.fused:
            # the INT8 path starts from the fp16 activations: every step quantizes them per token,
            # inside the matmul where the few-token kernel allows it
            wq.w4a8_gemm_fused(A, Wq, s, z, c.N, c.K, self.qc, out=C, out_q=self.Aq, out_scale=self.a_scale,
                               workspace=self.ws)
        else:
            wq.act_quant_int8(A, out_q=self.Aq, out_scale=self.a_scale)
            wq.w4a8_gemm(self.Aq, self.a_scale, Wq, s, z, c.N, c.K, self.qc, out=C, workspace=self.ws)


class StepIO:
    """End-to-end input / output staging.  Every case's activations sit in one pinned host
    buffer, and each step copies them in with one host-to-device copy. Every case's outputs
    are read back with one device-to-host copy per step.  The device buffers come in two
    slots (each case's A and C are 256-byte aligned views of them), and the copies run on
    their own stream.  Step s+1's inputs can then move while step s computes, and step s's
    results while step s+1 computes, as in a serving loop; a step's kernels wait for its own
    inputs only."""

    SLOTS = 2

    def __init__(self, preps, device):
        def layout(tensors):
            offs, total = [], 0
            for t in tensors:
                offs.append(total)
                total += (t.numel() * t.element_size() + 255) // 256 * 256
            return offs, total

        def views(buf, tensors, offs):
            return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(tensors, offs)]

        a_offs, a_total = layout([p.A for p in preps])
        c_offs, c_total = layout([p.C for p in preps])
        self.a_host = torch.zeros(a_total, dtype=torch.uint8).pin_memory()
        for hv, p in zip(views(self.a_host, [p.A for p in preps], a_offs), preps):
            hv.copy_(p.A_host)
        self.a_dev = [torch.zeros(a_total, dtype=torch.uint8, device=device) for _ in range(self.SLOTS)]
        self.c_dev = [torch.zeros(c_total, dtype=torch.uint8, device=device) for _ in range(self.SLOTS)]
        self.c_host = [torch.zeros(c_total, dtype=torch.uint8).pin_memory() for _ in range(self.SLOTS)]
        for sl in range(self.SLOTS):
            for p, av, cv in zip(preps, views(self.a_dev[sl], [p.A for p in preps], a_offs),
                                 views(self.c_dev[sl], [p.C for p in preps], c_offs)):
                if sl == 0:
                    p.A_slots, p.C_slots = [], []
                p.A_slots.append(av)
                p.C_slots.append(cv)
        self.h2d_bytes = a_total
        self.d2h_bytes = c_total
        self.stream = torch.cuda.Stream(device=device)
        self.ev = {k: [torch.cuda.Event() for _ in range(self.SLOTS)] for k in ("in", "done", "out")}
        self.fork = torch.cuda.Event()


def run_steps(preps, nsteps: int, e2e: bool, io=None):
    """`nsteps` steps, each running every case once.  End to end, each step's inputs are
    copied in from pinned host memory before its kernels and its results copied out after
    them, pipelined across steps on the copy stream (see StepIO); the launching stream waits
    for the last copy before it goes on."""
    if not e2e:
        for _ in range(nsteps):
            for p in preps:
                p.launch(False)
        return
    main, cs, ev, S = torch.cuda.current_stream(), io.stream, io.ev, StepIO.SLOTS
    io.fork.record(main)
    cs.wait_event(io.fork)
    with torch.cuda.stream(cs):
        io.a_dev[0].copy_(io.a_host, non_blocking=True)
    ev["in"][0].record(cs)
    for st in range(nsteps):
        sl = st % S
        main.wait_event(ev["in"][sl])
        if st >= S:
            main.wait_event(ev["out"][sl])  # step st - 2 has read this slot's outputs
        for p in preps:
            p.launch(True, sl)
        ev["done"][sl].record(main)
        if st + 1 < nsteps:  # the next step's inputs, once step st - 1 no longer reads that slot
            nx = (st + 1) % S
            if st >= 1:
                cs.wait_event(ev["done"][nx])
            with torch.cuda.stream(cs):
                io.a_dev[nx].copy_(io.a_host, non_blocking=True)
            ev["in"][nx].record(cs)
        cs.wait_event(ev["done"][sl])
        with torch.cuda.stream(cs):
            io.c_host[sl].copy_(io.c_dev[sl], non_blocking=True)
        ev["out"][sl].record(cs)
    main.wait_event(ev["out"][(nsteps - 1) % S])


def capture(preps, nsteps: int, e2e: bool, io=None):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_steps(preps, nsteps, e2e, io)
    return g


def timed_replays(preps, steps: int, warmup: int, e2e: bool, dist_on: bool, sampler=None, io=None):
    """Runs `warmup` untimed steps, then exactly `steps` timed steps; returns seconds (max over ranks)."""
    chunk = max(1, min(steps, 200))
    g_chunk = capture(preps, chunk, e2e, io)
    rem = steps % chunk
    g_rem = capture(preps, rem, e2e, io) if rem else None
    stream = torch.cuda.current_stream()
    # warm-up
    done = 0
    while done < warmup:
        n = min(chunk, warmup - done)
        if n == chunk:
            g_chunk.replay()
        else:
            run_steps(preps, n, e2e, io)
        done += n
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        t0.record(stream)
        for _ in range(steps // chunk):
            g_chunk.replay()
        if g_rem is not None:
            g_rem.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    sec = t0.elapsed_time(t1) / 1e3
    if dist_on:
        sec = max_over_ranks(sec, torch.device("cuda", torch.cuda.current_device()))
    del g_chunk, g_rem
    return sec


def max_over_ranks(sec: float, device=None) -> float:
    """The slowest rank's duration (every rank gets it); the local value without a process group."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return sec
    t = torch.tensor([sec], dtype=torch.float64, device=device if device is not None else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, steps: int, world: int, sec: float) -> float:
    """Units processed by all ranks together per second of the slowest rank (weak scaling)."""
    return units_per_step_per_rank * steps * world / sec


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass


def per_case_breakdown(preps, reps: int = 200):
    """Per-case microseconds (graph of `reps` launches of that case alone, events around it)."""
    out = []
    pk = peaks()
    for p in preps:
        g = capture([p], reps, False)
        g.replay()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        g.replay()
        t1.record()
        torch.cuda.synchronize()
        us = t0.elapsed_time(t1) * 1e3 / reps
        gbs = p.bytes / (us * 1e-6) / 1e9
        tf = flops(p.c) / (us * 1e-6) / 1e12
        peak_tc = pk["bf16_tflops"] * (2.0 if p.c.mode in ("a8", "f8") else 1.0)
        peak_tc_s = pk["bf16_tflops_sustained"] * (2.0 if p.c.mode in ("a8", "f8") else 1.0)
        t_roof = max(p.bytes / (pk["hbm_gbs"] * 1e9), flops(p.c) / (peak_tc * 1e12))
        out.append({"case": p.c.name, "us": round(us, 3), "GB/s": round(gbs, 1), "TFLOP/s": round(tf, 2),
                    "hbm_frac": round(gbs / pk["hbm_gbs"], 4), "tensor_frac": round(tf / peak_tc, 4),
                    "tensor_frac_sustained": round(tf / peak_tc_s, 4),
                    "roofline_frac": round(t_roof / (us * 1e-6), 4)})
        del g
    return out


# Workloads timed beside the headline one in the default run, each as its own object of the
# JSON line: the prefill GEMMs (the tensor-bound half of the metric), W4A8, the BitNet sweep
# and the other weight types (FP4, FP8, INT1) at decode and at prefill.
EXTRA_WORKLOADS = (("gemm", "prefill-llama7b"), ("w4a8", "w4a8"), ("bitnet3b", "bitnet3b"),
                   ("formats_decode", "formats-decode"), ("formats_prefill", "formats-prefill"))
TENSOR_BOUND = ("prefill-llama7b", "formats-prefill")


def measure_extra(name: str, device, steps: int, warmup: int, dist_on: bool) -> dict:
    """Device-timed steps of a further workload (same protocol as the headline), with its
    per-case breakdown and the roofline of its bound: the tensor peak (burst and sustained)
    for the prefill GEMMs, HBM bandwidth for the rest."""
    import gemv_wq_quantize_b200 as wq
    wl = wq_synth.WORKLOADS[name]
    preps = [Prepared(c, device, seed_base=0) for c in wl.cases]
    run_steps(preps, 1, False)
    torch.cuda.synchronize()
    sampler = ClockSampler(device)
    sec = timed_replays(preps, steps, warmup, False, dist_on, sampler)
    assert wq.device_error() == 0, "a kernel gave up a bounded wait"
    cases = per_case_breakdown(preps)
    step_bytes = sum(p.bytes for p in preps)
    step_flops = sum(flops(p.c) for p in preps)
    pk = peaks()
    gbs = step_bytes * steps / sec / 1e9
    tf = step_flops * steps / sec / 1e12
    out = {"workload": name, "description": wl.description, "steps": steps, "warmup": warmup,
           "ms_per_step": round(sec / steps * 1e3, 6), "GB/s": round(gbs, 2), "TFLOP/s": round(tf, 2),
           "gpu_launches": steps * sum(launches_per_call(p.c) for p in preps), "clocks": sampler.report()}
    if name in TENSOR_BOUND:
        out["roofline"] = {"bound": "tensor", "achieved": round(tf, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                           "frac": round(tf / pk["bf16_tflops"], 4), "peak_sustained": pk["bf16_tflops_sustained"],
                           "frac_sustained": round(tf / pk["bf16_tflops_sustained"], 4),
                           "traffic": recorded_traffic(name), "peak_source": pk["source"]}
    else:
        out["roofline"] = {"bound": "hbm", "achieved": round(gbs, 2), "peak": pk["hbm_gbs"], "unit": "GB/s",
                           "frac": round(gbs / pk["hbm_gbs"], 4), "traffic": recorded_traffic(name),
                           "peak_source": pk["source"]}
    out["cases"] = cases
    if any(p.c.mode in ("a8", "f8") for p in preps):
        # the same INT8 cases with the activation quantization as a kernel of its own
        for p in preps:
            p.fused = False
        run_steps(preps, 1, False)
        torch.cuda.synchronize()
        out["cases_two_launches"] = [c for c, p in zip(per_case_breakdown(preps), preps) if p.c.mode in ("a8", "f8")]
    del preps
    torch.cuda.empty_cache()
    return out


LLAMA7B_LAYER = (("qkv", 12288, 4096), ("o", 4096, 4096), ("gate_up", 22016, 4096), ("down", 4096, 11008))


def measure_layer_graph(device, M: int = 1, reps: int = 50) -> dict:
    """One Llama-7B layer's four decode projections (asymmetric INT4, group 128, fp16) over
    enough layer copies (6 x 107 MB) that every launch streams its weights from HBM, run as one
    wq_graph (built once; one launch per pass over the layers).  Reported per layer: the
    wq_graph, the same kernels captured by torch stream capture, and four direct C-ABI calls
    per layer issued from this Python process."""
    import gemv_wq_quantize_b200 as wq
    qc = wq.QuantConfig(4, 128, False)
    base = []
    for i, (name, N, K) in enumerate(LLAMA7B_LAYER):
        Wq, s, z = wq.quantize_pack(wq_synth.weights(N, K, seed=i).to(device), qc)
        A = wq_synth.activations(M, K, seed=10 + i, outlier_frac=0.01).to(device)
        C = torch.empty(M, N, dtype=torch.float16, device=device)
        base.append((name, N, K, Wq, s, z, A, C))
    layer_bytes = sum(alg_bytes(wq_synth.Case(M, N, K, "a16", "asym4")) for _, N, K, *_ in base)
    nlayers = max(2, math.ceil(4 * L2_BYTES / layer_bytes) + 1)
    layers = [[(name, N, K, Wq.clone(), s.clone(), z.clone(), A, C) for name, N, K, Wq, s, z, A, C in base]
              for _ in range(nlayers)]
    # one graph over all layer copies (a decode step runs its layers back to back)
    graph = wq.DecodeGraph([{"A": A, "Wq": Wq, "scales": s, "zeros": z, "N": N, "K": K, "qc": qc, "out": C}
                            for layer in layers for _, N, K, Wq, s, z, A, C in layer])

    def calls():
        for layer in layers:
            for _, N, K, Wq, s, z, A, C in layer:
                wq.w4a16_gemm(A, Wq, s, z, N, K, qc, out=C)

    def timed(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(n):
            fn()
        t1.record()
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) * 1e3 / (n * nlayers)

    us_graph = timed(graph.launch, reps)

    def host_us(fn, n):  # host time to enqueue one pass (no synchronisation inside)
        torch.cuda.synchronize()
        t = time.perf_counter()
        for _ in range(n):
            fn()
        dt = time.perf_counter() - t
        torch.cuda.synchronize()
        return dt * 1e6 / (n * nlayers)

    host_graph = host_us(graph.launch, 20)
    host_calls = host_us(calls, 5)
    cap = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cap):
        calls()
    us_captured = timed(cap.replay, reps)
    us_calls = timed(calls, max(5, reps // 5))
    graph.close()
    assert wq.device_error() == 0, "a kernel gave up a bounded wait"
    pk = peaks()
    return {"ops": [f"{n}:{N}x{K}" for n, N, K in LLAMA7B_LAYER], "M": M, "layer_copies": nlayers,
            "bytes_per_layer": layer_bytes, "us_per_layer_graph": round(us_graph, 3),
            "us_per_layer_stream_captured": round(us_captured, 3), "us_per_layer_direct_calls": round(us_calls, 3),
            "host_us_per_layer_graph": round(host_graph, 3), "host_us_per_layer_direct_calls": round(host_calls, 3),
            "GB/s_graph": round(layer_bytes / (us_graph * 1e-6) / 1e9, 1),
            "hbm_frac_graph": round(layer_bytes / (us_graph * 1e-6) / 1e9 / pk["hbm_gbs"], 4)}


def measure_native(name: str, device) -> list:
    """Per-case times of a workload's INT4 cases with the weights in the kernel-native order
    (wq_repack), to set beside the same cases on the "nt" packing."""
    wl = wq_synth.WORKLOADS[name]
    preps = [Prepared(c, device, seed_base=0, native=True) for c in wl.cases if c.quant != "tern2"]
    run_steps(preps, 1, False)
    torch.cuda.synchronize()
    out = per_case_breakdown(preps)
    del preps
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank, dist_on):
    import gemv_wq_quantize_b200 as wq
    from gemv_wq_quantize_b200 import build
    build.build(quiet=True)
    wq.load_library()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    wl = wq_synth.WORKLOADS[args.workload]
    preps = [Prepared(c, device, seed_base=0) for c in wl.cases]
    io = StepIO(preps, device)
    run_steps(preps, 1, False)   # first calls configure the kernels outside any capture
    run_steps(preps, 2, True, io)
    torch.cuda.synchronize()
    sampler = ClockSampler(device)
    sec = timed_replays(preps, args.steps, args.warmup, False, dist_on, sampler)
    sec_e2e = timed_replays(preps, args.steps, args.warmup, True, dist_on, io=io)
    assert wq.device_error() == 0, "a kernel gave up a bounded wait"
    step_bytes = sum(p.bytes for p in preps)
    step_flops = sum(flops(p.c) for p in preps)
    launches = sum(launches_per_call(p.c) for p in preps)
    value = whole_job_rate(step_bytes, args.steps, world, sec) / 1e9
    e2e_value = whole_job_rate(step_bytes, args.steps, world, sec_e2e) / 1e9
    pk = peaks()
    avg_launch_s = sec / (args.steps * launches)
    achieved = (step_bytes / launches) / avg_launch_s / 1e9
    achieved_tf = (step_flops / launches) / avg_launch_s / 1e12
    tensor_bound = args.workload == "prefill-llama7b"
    result = {
        "metric": "W4 GEMV GB/s & GEMM TFLOP/s at 1 B200; fraction of HBM / tensor roofline",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec / args.steps * 1e3, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16" if not tensor_bound else "bf16", "weight_dtype": "int4" if
        "tern" not in args.workload else "int2",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) activations, 1% outlier channels x20)",
        "config": {"workload": wl.name, "description": wl.description,
                   "cases": [p.c.name for p in preps],
                   "l2": "inputs larger than L2: each case rotates over >= 4x126MB of weight copies",
                   "timing": "CUDA graphs of whole steps, CUDA events on the launch stream, max over ranks"},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": io.h2d_bytes, "d2h_bytes_per_step": io.d2h_bytes},
        "gpu_launches": args.steps * (launches + 0),
        "roofline": ({"bound": "tensor", "achieved": round(achieved_tf, 2), "peak": pk["bf16_tflops"],
                      "unit": "TFLOP/s", "frac": round(achieved_tf / pk["bf16_tflops"], 4),
                      "traffic": recorded_traffic(args.workload), "peak_source": pk["source"]} if tensor_bound else
                     {"bound": "hbm", "achieved": round(achieved, 2), "peak": pk["hbm_gbs"], "unit": "GB/s",
                      "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": recorded_traffic(args.workload),
                      "peak_source": pk["source"]}),
        "tflops": round(step_flops * args.steps * world / sec / 1e12, 3),
        "clocks": sampler.report(),
    }
    if not args.no_breakdown:
        result["cases"] = per_case_breakdown(preps)
    del preps, io
    torch.cuda.empty_cache()
    if args.workload == "decode-llama7b" and not args.no_extra:
        for key, name in EXTRA_WORKLOADS:
            result[key] = measure_extra(name, device, min(args.steps, 2000), args.warmup, dist_on)
        result["decode_layer_graph"] = measure_layer_graph(device)
        result["native_layout"] = {"note": "the same cases with the weights repacked into the kernel-native order",
                                   "decode-llama7b": measure_native("decode-llama7b", device),
                                   "prefill-llama7b": measure_native("prefill-llama7b", device)}
    return result


# ------------------------------------------------------------------ oracle timing
def oracle_sample(wl, budget_s: float, threads: int):
    """Runs the CPU oracle on a bounded sample of every case (a subset of output columns,
    all tokens) and returns (algorithmic bytes covered, seconds, description)."""
    import oracle
    oracle.build()
    prepared = []
    max_frac = 1.0 / 16  # the sample never covers more output columns than this
    for c in wl.cases:
        # only the weight rows a sample can use are quantized (codes and group scales are
        # per row; the per-tensor scale of INT2 / INT1 then comes from these rows)
        W = wq_synth.weights(c.N, c.K, seed=0).numpy()[:max(1, math.ceil(c.N * max_frac))]
        A = wq_synth.activations(c.M, c.K, seed=1, dtype=c.a_dtype, outlier_frac=c.outlier_frac)
        Abits = A.contiguous().view(torch.int16).numpy().view(np.uint16)
        fmt = oracle.FMT_INT
        if c.quant == "tern2":
            Wq, s = oracle.quantize_ternary(W)
            z, bits, sym = None, 2, True
        elif c.quant == "int1":
            Wq, s = oracle.quantize_binary(W)
            z, bits, sym = None, 1, True
        elif c.quant in ("e2m1", "e4m3"):
            fmt = oracle.FMT_E2M1 if c.quant == "e2m1" else oracle.FMT_E4M3
            Wq, s = oracle.quantize_minifloat(W, c.group_size, fmt)
            z, bits, sym = None, wq_synth.QUANT_BITS[c.quant], True
        else:
            Wq, s, z = oracle.quantize_int4(W, c.group_size, c.quant == "sym4")
            bits, sym = 4, c.quant == "sym4"
        prepared.append((c, Abits, Wq, s, z, bits, sym, fmt))

    def run(frac):
        t = 0.0
        covered = 0.0
        for c, Abits, Wq, s, z, bits, sym, fmt in prepared:
            rows = Wq.shape[0]
            n_cnt = min(rows, max(1, int(round(c.N * frac))))
            ni = np.arange(n_cnt)
            t0 = time.perf_counter()
            if c.mode == "a16":
                adt = oracle.F16 if c.a_dtype == torch.float16 else oracle.BF16
                oracle.gemm_a16(Abits, adt, Wq, rows, c.K, bits, sym, c.group_size, s, z, n_idx=ni, threads=threads,
                                fmt=fmt)
            elif c.mode == "f8":
                Aq, asc = oracle.act_quant_e4m3(Abits, oracle.F16)
                oracle.gemm_f8(Aq, asc, Wq, rows, c.K, c.group_size, s, n_idx=ni, threads=threads)
            else:
                Aq, asc = oracle.act_quant_int8(Abits, oracle.F16)
                oracle.gemm_a8(Aq, asc, Wq, rows, c.K, bits, sym, c.group_size, s, z, n_idx=ni, threads=threads)
            t += time.perf_counter() - t0
            covered += alg_bytes(c) * n_cnt / c.N
        return covered, t

    frac = 1.0 / 512
    covered, t = run(frac)
    if t < budget_s / 4:
        frac = min(max_frac, frac * budget_s / max(t, 1e-3) / 2)
        covered, t = run(frac)
    desc = f"oracle on {frac:.4%} of the output columns of every case (all tokens), {threads} threads"
    return covered, t, desc


def run_reference(args):
    wl = wq_synth.WORKLOADS[args.workload]
    threads = os.cpu_count() or 1
    budget = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wl, budget / 4, threads)
    covered = secs = 0.0
    desc = ""
    for _ in range(args.steps):
        cb, s, desc = oracle_sample(wl, budget, threads)
        covered += cb
        secs += s
    v = covered / secs / 1e9
    return {"metric": "W4 GEMV GB/s & GEMM TFLOP/s at 1 B200; fraction of HBM / tensor roofline",
            "value": round(v, 6), "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "description": wl.description},
            "cpu_baseline": {"value": round(v, 6), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_profile(args):
    """One plain launch per case (one weight copy each; ncu flushes the caches itself)."""
    import gemv_wq_quantize_b200 as wq
    from gemv_wq_quantize_b200 import build
    build.build(quiet=True)
    wq.load_library()
    device = torch.device("cuda", 0)
    wl = wq_synth.WORKLOADS[args.workload]
    preps = [Prepared(c, device, seed_base=0, copies=1) for c in wl.cases]
    torch.cuda.synchronize()
    for p in preps:
        p.launch(False)
    torch.cuda.synchronize()
    assert wq.device_error() == 0, "a kernel gave up a bounded wait"
    print(json.dumps({"profile": wl.name, "cases": [p.c.name for p in preps],
                      "source_sha": kernel_source_hash()}), flush=True)


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="decode-llama7b", choices=sorted(wq_synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the chosen workload (the default run adds the prefill GEMM, W4A8 and BitNet)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--profile", action="store_true",
                    help="launch each case of the workload once, untimed (the command an ncu capture wraps)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.profile:
        run_profile(args)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    dist_on = world > 1
    if dist_on:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    result = run_ours(args, rank, world, local_rank, dist_on)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl = wq_synth.WORKLOADS[args.workload]
        threads = os.cpu_count() or 1
        covered, secs, desc = oracle_sample(wl, args.cpu_budget, threads)
        result["cpu_baseline"] = {"value": round(covered / secs / 1e9, 6), "unit": "GB/s", "cores": threads,
                                  "kind": "oracle", "sample": desc}
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


if __name__ == "__main__":
    main()
