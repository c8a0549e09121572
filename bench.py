"""Benchmark of the SSA dual-stream attention layer on B200.

One step = the whole hot path over one batch of synthetic input, through the
C ABI: block selection -> fused dual-stream forward -> alignment loss ->
backward of both streams (upstream N(0,1) gradients on both outputs plus
both alignment terms).  Default workload: B=1, H=16, T=8192, d=128, bf16,
block 64, top-k 16 with planted hot blocks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is algorithmic TFLOP/s of the step
(forward 4*d*P_full, backward 10*d*P_full + 4*d*P_sel per head, P_full =
T(T+1)/2 causal pairs, P_sel = selected causal pairs) summed over all ranks,
divided by the slowest rank's device time; inputs are resident in HBM and L2
is flushed before every timed step.  Under torchrun each rank runs its own
copy of the workload (independent (batch, head) units, no data-path
collective): weak scaling.

``--impl reference`` times the fp64 CPU oracle on a bounded slice of the
same workload on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import ctypes
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_full_b200.inputs import WORKLOADS, Workload, make_inputs, upstream_grads  # noqa: E402

DEFAULT_WORKLOAD = "bf16_T8192_H16_hot"
METRIC = "dual-stream SSA attention fwd(+bwd) TFLOP/s and % bf16 tensor peak at T=8192"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
FP32_LANES_PER_SM = 128
NUM_SMS = 148
SPEC_BF16_TFLOPS = 2250.0  # B200 dense bf16 data-sheet figure, for context
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def pair_counts(w, idx, cnt):
    """Causal pairs per (b, h): full = T(T+1)/2 and selected (from idx/cnt)."""
    T, blk = w.T, w.block
    p_full = T * (T + 1) // 2
    idx = idx.reshape(-1, w.n_blocks, idx.shape[-1])
    cnt = cnt.reshape(-1, w.n_blocks)
    p_sel = 0
    for bh in range(idx.shape[0]):
        for i in range(w.n_blocks):
            js = idx[bh, i, :cnt[bh, i]]
            # rows of block i see all keys of earlier selected blocks and the
            # causal triangle of block i itself
            p_sel += blk * blk * int((js < i).sum()) + blk * (blk + 1) // 2
    return p_full, p_sel / idx.shape[0]


def step_flops(w, p_full, p_sel):
    BH = w.B * w.H
    f_fwd = 4 * w.D * p_full * BH
    f_bwd = (10 * w.D * p_full + 4 * w.D * p_sel) * BH
    return f_fwd, f_bwd


def kernel_flops(w, p_full, p_sel):
    """Algorithmic FLOPs of each tensor-core kernel of one step.  fwd: S and
    P V of the full stream (the sparse stream's products are a subset of the
    same tiles); dK/dV kernel: S^T, dP_f^T, dV, dK per causal pair plus dP_s^T
    and the sparse dV per selected pair; dQ GEMM: dS K per causal pair."""
    BH, d = w.B * w.H, w.D
    return {"fwd_tc_kernel": 4 * d * p_full * BH,
            "bwd_dkdv_tc_kernel": (8 * d * p_full + 4 * d * p_sel) * BH,
            "bwd_dq_gemm_kernel": 2 * d * p_full * BH}


def ds_blocks_per_bh(T):
    """[128 keys x 64 queries] dS^T blocks of the causal triangle of one head."""
    ntk = (T + 127) // 128
    return ntk * (T // 64) - ntk * (ntk - 1)


def workload_config(w, world, parallelism):
    """The ``config`` object both arms print for workload ``w``."""
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "D": w.D, "block": w.block,
            "topk": w.topk, "global_batch": w.B * world, "seq_len": w.T,
            "parallelism": parallelism}


def data_description(w):
    """What the synthetic inputs of workload ``w`` are, for the JSON line."""
    base = "synthetic (seeded N(0,1)" + ("/sqrt(d)" if w.scale_data else "")
    if w.plant == "hot":
        return base + f", {w.n_hot} planted hot key blocks per head)"
    if w.plant == "sink":
        return base + ", a planted heavy sink in key block 0)"
    return base + ")"


def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "block_sparse_full_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """DRAM bytes per launch recorded from an ncu capture of this kernel on
    this workload, or None when no such capture exists or the kernel source
    changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    e = table.get(kernel_key)
    if not e or e.get("source_sha") != source_sha(*e["sources"]):
        return None
    if e.get("workload", "").split(" ")[0] != workload:
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event reasons while the timed region runs: NVML read
    every 5 ms from a thread (reads only, no setting is changed), plus
    nvidia-smi at 200 ms as a second source."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h): sw power cap, hw slowdown, sw/hw thermal
    NVML_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                 "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None
        self.nvml = []
        self._stop = None
        self._thread = None

    def _nvml_loop(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            while not self._stop.is_set():
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                self.nvml.append((sm, mx, get_reasons(h)))
                self._stop.wait(0.005)
            pynvml.nvmlShutdown()
        except Exception:  # NVML unavailable: nvidia-smi samples only
            pass

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._nvml_loop, daemon=True)
        self._thread.start()
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for c, m, bits in self.nvml:
            sm.append(float(c))
            mx.append(float(m))
            reasons.update(n for n, bit in self.NVML_BITS.items() if bits & bit)
        src = "nvml" if sm else None
        if self.file is not None:
            self.file.flush()
            with open(self.file.name) as f:
                rows = [r.split(",") for r in f.read().strip().splitlines() if r.strip()]
            os.unlink(self.file.name)
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for r in rows:
                try:
                    c, m = float(r[1]), float(r[2])
                except (ValueError, IndexError):
                    continue
                sm.append(c)
                mx.append(m)
                reasons.update(n for n, v in zip(names, r[4:8]) if v.strip().lower() == "active")
                src = "nvml+nvidia-smi" if src else "nvidia-smi"
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm), "source": src}


# ----------------------------------------------------------------------------- our arm

class Layer:
    """Preallocated device buffers and raw C-ABI calls for one step."""

    def __init__(self, w, inp, grads, dev):
        from block_sparse_full_b200 import ssa
        self.ssa, self.w, self.dev = ssa, w, dev
        self.q, self.k, self.v = (inp[n].to(dev) for n in "qkv")
        self.dhf, self.dhs = grads["dh_full"].to(dev), grads["dh_sparse"].to(dev)
        self.p = ssa.params_for(self.q, w.block, w.topk, w.sm_scale, w.flags)
        n, words = w.n_blocks, (w.n_blocks + 31) // 32
        B, H, T = w.B, w.H, w.T
        self.idx = torch.empty((B, H, n, w.topk), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, H, n), dtype=torch.int32, device=dev)
        self.mask = torch.empty((B, H, n, words), dtype=torch.int32, device=dev)
        self.hf, self.hs = torch.empty_like(self.q), torch.empty_like(self.q)
        self.rows = {k: torch.empty((B, H, T), dtype=torch.float32, device=dev)
                     for k in ("delta", "lse_f", "lse_s", "sqd")}
        self.loss = torch.empty(2, dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
        self.ws = {i: ssa.workspace(self.p, i, dev) for i in range(5)}
        self.sink = torch.empty((B, H, T), dtype=torch.float32, device=dev)  # diagnostics
        self.head_stats = torch.empty((B, H, 2), dtype=torch.float32, device=dev)
        self.hs_inf = torch.empty_like(self.q)  # sparse-only forward (inference) outputs
        self.ls_inf = torch.empty((B, H, T), dtype=torch.float32, device=dev)
        self.w_s = self.w_c = 1.0
        self.path = ssa.ssa_kernel_path(self.p)

    def launches_per_step(self):
        # select: pool + score; fwd: 1; loss: 2; bwd: pre + dk/dv + dq on the
        # tensor-core path, pre + one dq-and-dk/dv grid on the CUDA-core path
        return 2 + 1 + 2 + (3 if self.path == 1 else 2)

    def run_sparse_fwd(self, stream):
        """The sparse stream alone (inference mode) on the step's selection."""
        ssa, ptr = self.ssa, (lambda t: t.data_ptr())
        st = ssa.ssa_attn_fwd_sparse(self.p, ptr(self.q), ptr(self.k), ptr(self.v), None, None,
                                     ptr(self.mask), ptr(self.hs_inf), ptr(self.ls_inf),
                                     ptr(self.ws[4]), self.ws[4].numel(), stream.cuda_stream)
        ssa.check(st, "sparse fwd")

    def run_diagnostics(self, stream):
        """Sink mass on block 0 and per-head means, from the step's forward outputs."""
        ssa, ptr, r = self.ssa, (lambda t: t.data_ptr()), self.rows
        st = ssa.ssa_attn_diagnostics(self.p, ptr(self.q), ptr(self.k), ptr(r["lse_f"]),
                                      ptr(r["delta"]), ptr(self.sink), ptr(self.head_stats),
                                      stream.cuda_stream)
        ssa.check(st, "diagnostics")

    def run_fwd_diag(self, stream):
        """The dual forward with the diagnostics folded in (one call)."""
        ssa, ptr, r = self.ssa, (lambda t: t.data_ptr()), self.rows
        st = ssa.ssa_attn_fwd_dual_diag(self.p, ptr(self.q), ptr(self.k), ptr(self.v), None, None,
                                        ptr(self.mask), ptr(self.hf), ptr(self.hs), ptr(r["delta"]),
                                        ptr(r["lse_f"]), ptr(r["lse_s"]), ptr(r["sqd"]),
                                        ptr(self.sink), ptr(self.head_stats), ptr(self.ws[1]),
                                        self.ws[1].numel(), stream.cuda_stream)
        ssa.check(st, "fwd + diagnostics")

    def run(self, stream, events=None, kernel_events=None):
        """One step; `events` (5) bracket the four ABI calls, `kernel_events`
        (4, tensor-core path) the kernels inside the backward call."""
        s, ssa, P = stream.cuda_stream, self.ssa, self.p
        ptr = lambda t: t.data_ptr()
        ev = events or [None] * 5
        if ev[0] is not None:
            ev[0].record(stream)
        st = ssa.ssa_select_blocks(P, ptr(self.q), ptr(self.k), ptr(self.idx), ptr(self.cnt),
                                   ptr(self.mask), ptr(self.ws[0]), self.ws[0].numel(), s)
        ssa.check(st, "select")
        if ev[1] is not None:
            ev[1].record(stream)
        r = self.rows
        st = ssa.ssa_attn_fwd_dual(P, ptr(self.q), ptr(self.k), ptr(self.v), None, None,
                                   ptr(self.mask), ptr(self.hf), ptr(self.hs), ptr(r["delta"]),
                                   ptr(r["lse_f"]), ptr(r["lse_s"]), ptr(r["sqd"]),
                                   ptr(self.ws[1]), self.ws[1].numel(), s)
        ssa.check(st, "fwd")
        if ev[2] is not None:
            ev[2].record(stream)
        st = ssa.ssa_align_loss(P, ptr(r["sqd"]), self.w_s, self.w_c, ptr(self.loss),
                                ptr(self.ws[2]), self.ws[2].numel(), s)
        ssa.check(st, "loss")
        if ev[3] is not None:
            ev[3].record(stream)
        if kernel_events is not None:
            handles = (ctypes.c_void_p * 4)(*[e.cuda_event for e in kernel_events])
            ssa.check(ssa.ssa_debug_set_kernel_events(handles, 4), "kernel events")
        st = ssa.ssa_attn_bwd(P, ptr(self.q), ptr(self.k), ptr(self.v), None, None,
                              ptr(self.mask), ptr(self.hf), ptr(self.hs), ptr(r["lse_f"]),
                              ptr(r["lse_s"]), ptr(self.dhf), ptr(self.dhs), self.w_s, self.w_c,
                              ptr(self.dq), ptr(self.dk), ptr(self.dv), ptr(self.ws[3]),
                              self.ws[3].numel(), s)
        if kernel_events is not None:
            ssa.ssa_debug_set_kernel_events(None, 0)
        ssa.check(st, "bwd")
        if ev[4] is not None:
            ev[4].record(stream)


def run_ours(args, rank, world, dev, peaks, peak_src):
    w = workload(args)
    torch.cuda.set_device(dev)
    inp = make_inputs(w)
    grads = upstream_grads(w)
    layer = Layer(w, inp, grads, dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    for _ in range(args.warmup):
        layer.run(stream)
    torch.cuda.synchronize(dev)
    layer.ssa.device_status()
    p_full, p_sel = pair_counts(w, layer.idx.cpu().numpy(), layer.cnt.cpu().numpy())
    f_fwd, f_bwd = step_flops(w, p_full, p_sel)

    names = ("select", "fwd", "loss", "bwd")
    per_call = {n: 0.0 for n in names}
    step_ms = []
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    kevs = None
    if layer.path == 1:  # per-kernel events inside the backward call
        kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        for ks in kevs:
            for e in ks:
                e.record(stream)  # creates the event so its handle can be passed down
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush.zero_()  # evict L2 between timed steps (outside the events)
            layer.run(stream, evs[i], kevs[i] if kevs else None)
        torch.cuda.synchronize(dev)
    barrier(world)
    layer.ssa.device_status()
    for e in evs:
        step_ms.append(e[0].elapsed_time(e[4]))
        for j, n in enumerate(names):
            per_call[n] += e[j].elapsed_time(e[j + 1])
    total_ms = sum(step_ms)
    max_ms = reduce_max(total_ms, world, dev)
    ms_per_step = max_ms / args.steps
    value = whole_job_tflops(f_fwd + f_bwd, world, ms_per_step)

    # per-kernel times (fwd: the call is its one kernel) and the dominant kernel's roofline
    avg = {n: per_call[n] / args.steps for n in names}
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # the yardstick matches the timed region: a region under a second runs
    # like the burst GEMM measurement, a longer one like the sustained loop
    peak, peak_kind = roofline_peak(total_ms, burst, sustained)
    kernels = None
    if layer.path == 1:
        kms = {"fwd_tc_kernel": avg["fwd"], "bwd_tc_pre_kernel": 0.0, "bwd_dkdv_tc_kernel": 0.0,
               "bwd_dq_gemm_kernel": 0.0}
        for ks in kevs:
            kms["bwd_tc_pre_kernel"] += ks[0].elapsed_time(ks[1]) / args.steps
            kms["bwd_dkdv_tc_kernel"] += ks[1].elapsed_time(ks[2]) / args.steps
            kms["bwd_dq_gemm_kernel"] += ks[2].elapsed_time(ks[3]) / args.steps
        kfl = kernel_flops(w, p_full, p_sel)
        # the events bracket the backward kernels of the first group of heads
        group = layer.ssa.ssa_bwd_heads_per_group(layer.p) / (w.B * w.H)
        for k in ("bwd_dkdv_tc_kernel", "bwd_dq_gemm_kernel"):
            kfl[k] *= group
        kernels = {k: {"ms": round(v, 4)} for k, v in kms.items()}
        kernels["bwd_heads_per_group"] = layer.ssa.ssa_bwd_heads_per_group(layer.p)
        for k, f in kfl.items():
            kernels[k]["tflops"] = round(f / (kms[k] * 1e-3) / 1e12, 2)
        # the dQ GEMM streams the stored dS^T blocks: its own bound is HBM
        dq_bytes = round((ds_blocks_per_bh(w.T) * 64 * 128 * 2 + 2 * w.T * w.D * 2) * w.B * w.H * group)
        kernels["bwd_dq_gemm_kernel"]["hbm_gbs"] = round(dq_bytes / (kms["bwd_dq_gemm_kernel"] * 1e-3) / 1e9, 1)
        kernels["bwd_dq_gemm_kernel"]["hbm_bytes"] = dq_bytes
        dom = max(kfl, key=lambda k: kms[k])
        roof = {"kernel": dom, "bound": "tensor", "peak": peak, "unit": "TFLOP/s",
                "peak_kind": f"{peak_src} bf16 dense, {peak_kind}", "traffic": ncu_traffic(dom, w.name)}
        flops, dom_ms = kfl[dom], kms[dom]
    else:
        dom = max(("fwd", "bwd"), key=lambda n: avg[n])
        flops = f_fwd if dom == "fwd" else f_bwd
        fp32 = NUM_SMS * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        roof = {"kernel": f"{dom}_simt", "bound": "alu", "peak": round(fp32, 1),
                "unit": "TFLOP/s", "peak_kind": "fp32 FMA: 148 SMs x 128 lanes x 2 x max SM clock",
                "traffic": ncu_traffic(f"{dom}_simt", w.name)}
        dom_ms = avg[dom]
    achieved = flops / (dom_ms * 1e-3) / 1e12
    roof["achieved"] = round(achieved, 2)
    roof["frac"] = round(achieved / roof["peak"], 4)
    if roof["bound"] == "tensor":
        roof["frac_of_sustained"] = round(achieved / sustained, 4)
        roof["timed_region_ms"] = round(total_ms, 2)
    roof["ms_per_launch"] = round(dom_ms, 4)
    roof["flops_per_launch"] = flops

    # inference mode: the sparse stream alone on the same selection (not part
    # of the training step; timed after it, L2 flushed before each call)
    inf_ms = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer.run_sparse_fwd(stream)
        e1.record(stream)
        if i >= args.warmup:
            inf_ms.append((e0, e1))
    torch.cuda.synchronize(dev)
    layer.ssa.device_status()
    sparse_ms = sum(a.elapsed_time(b) for a, b in inf_ms) / len(inf_ms)
    diag_ev = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer.run_diagnostics(stream)
        e1.record(stream)
        if i >= args.warmup:
            diag_ev.append((e0, e1))
    torch.cuda.synchronize(dev)
    layer.ssa.device_status()
    diag_ms = sum(a.elapsed_time(b) for a, b in diag_ev) / len(diag_ev)
    # the forward with the diagnostics folded in, against the forward alone
    fused_ev = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer.run_fwd_diag(stream)
        e1.record(stream)
        if i >= args.warmup:
            fused_ev.append((e0, e1))
    torch.cuda.synchronize(dev)
    layer.ssa.device_status()
    fused_ms = sum(a.elapsed_time(b) for a, b in fused_ev) / len(fused_ev)
    decode = decode_bench(args, w, layer, stream, flush, dev)

    # reads Q, block 0 of K, lse_full and delta; writes the sink row vector
    esz = 2 if w.dtype == "bf16" else 4
    diag_bytes = w.B * w.H * (w.T * w.D * esz + min(w.block, w.T) * w.D * esz + 3 * w.T * 4)
    hs = layer.head_stats.cpu().numpy()
    diagnostics = {"kernels": ["diag_sink_kernel", "diag_head_kernel"], "ms": round(diag_ms, 4),
                   "fwd_with_diagnostics_ms": round(fused_ms, 4),
                   "fused_adds_over_fwd_ms": round(fused_ms - avg["fwd"], 4),
                   "hbm_bytes": diag_bytes, "hbm_gbs": round(diag_bytes / (diag_ms * 1e-3) / 1e9, 1),
                   "mean_delta": round(float(hs[..., 0].mean()), 6),
                   "mean_sink_mass": round(float(hs[..., 1].mean()), 6)}
    f_sparse = 4 * w.D * p_sel * w.B * w.H
    inference = {"kernel": "fwd_tc_kernel<sparse>" if layer.path == 1 else "fwd_simt (dual)",
                 "ms": round(sparse_ms, 4), "flops": f_sparse,
                 "tflops": round(f_sparse / (sparse_ms * 1e-3) / 1e12, 2),
                 "dual_fwd_ms": round(avg["fwd"], 4),
                 "speedup_vs_dual_fwd": round(avg["fwd"] / sparse_ms, 3)}

    fwd_tflops = f_fwd / (avg["fwd"] * 1e-3) / 1e12
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": data_description(w),
        "config": {**workload_config(w, world, f"replicas x{world} (independent batch*head units)"),
                   "l2": "flushed before every timed step", "kernel_path": layer.path},
        "roofline": roof,
        "breakdown_ms": {n: round(avg[n], 4) for n in names},
        "kernels": kernels,
        "inference_sparse_fwd": inference,
        "diagnostics": diagnostics,
        "decode_step": decode,
        "fwd_tflops": round(fwd_tflops, 2),
        "fwd_frac_burst": round(fwd_tflops / burst, 4),
        "fwd_frac_sustained": round(fwd_tflops / sustained, 4),
        "fwd_frac_spec": round(fwd_tflops / SPEC_BF16_TFLOPS, 4),
        "flops_per_step": {"fwd": f_fwd, "bwd": f_bwd, "P_full": p_full, "P_sel": p_sel},
        "gpu_launches": layer.launches_per_step() * args.steps,
        "clocks": clk.summary(),
        "peaks": {"source": peak_src, "bf16_tflops": peaks.get("bf16_tflops"),
                  "bf16_tflops_sustained": sustained, "hbm_gbs": peaks.get("hbm_gbs")},
    }
    if args.e2e:
        out["e2e"] = run_e2e(args, layer, inp, grads, f_fwd + f_bwd, world, dev)
    if args.long_context and layer.path == 1:
        del layer, inp, grads  # the step's buffers are not needed any more
        torch.cuda.empty_cache()
        out["long_context_128k"] = long_context_bench(args, stream, flush, dev)
    return out


def run_e2e(args, layer, inp, grads, flops, world, dev):
    """Same metric with host buffers: every step copies its inputs from pinned
    host memory to the device and reads the loss back, inside the timing.

    The inputs are double-buffered: while step i runs on one set of device
    buffers, a copy stream fills the other with step i+1's inputs (as a
    training loop prefetches its next batch).  Events order each copy after
    the last step that read its buffers, and each step after its copies."""
    host = {n: inp[n].pin_memory() for n in "qkv"}
    host["dh_full"] = grads["dh_full"].pin_memory()
    host["dh_sparse"] = grads["dh_sparse"].pin_memory()
    loss_h = torch.empty(2, dtype=torch.float32).pin_memory()
    attr = {"q": "q", "k": "k", "v": "v", "dh_full": "dhf", "dh_sparse": "dhs"}
    sets = [{n: getattr(layer, a) for n, a in attr.items()},
            {n: torch.empty_like(getattr(layer, a)) for n, a in attr.items()}]
    stream = torch.cuda.current_stream(dev)
    copier = torch.cuda.Stream(dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    used = [torch.cuda.Event(), torch.cuda.Event()]
    used[0].record(stream)
    used[1].record(stream)

    def copy_in(i):
        b = i & 1
        copier.wait_event(used[b])  # the step that last read these buffers is done
        with torch.cuda.stream(copier):
            for n, t in host.items():
                sets[b][n].copy_(t, non_blocking=True)
        copied[b].record(copier)

    def compute(i):
        b = i & 1
        for n, a in attr.items():
            setattr(layer, a, sets[b][n])
        stream.wait_event(copied[b])
        layer.run(stream)
        loss_h.copy_(layer.loss, non_blocking=True)
        used[b].record(stream)

    def steps(k):
        copy_in(0)
        for i in range(k):
            if i + 1 < k:
                copy_in(i + 1)
            compute(i)

    steps(max(1, args.warmup))
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copier.wait_event(e0)  # the first copy starts inside the timed region
    steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    for n, a in attr.items():  # the layer keeps its own buffers afterwards
        setattr(layer, a, sets[0][n])
    ms = reduce_max(e0.elapsed_time(e1), world, dev) / args.steps
    return {"value": round(whole_job_tflops(flops, world, ms), 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": loss_h.numel() * loss_h.element_size(),
            "overlap": "step i+1's host-to-device copies on a second stream during step i"}


# ----------------------------------------------------------------------------- oracle arm

def oracle_slice(w, inp, grads, sel, row_slice):
    """Oracle select + forward + loss + backward for head (0, 0) restricted
    to the query rows ``row_slice``; returns (algorithmic flops, seconds)."""
    from oracle import ssa_oracle as O
    q, k, v = (inp[n][:1, :1] for n in "qkv")
    rows = np.arange(row_slice.start, row_slice.stop)
    t0 = time.perf_counter()
    idx, cnt, _, _ = O.select_blocks(q, k, w.block, w.topk)
    fw = O.attn_fwd_dual(q, k, v, idx, cnt, w.block, w.sm_scale, rows=rows)
    O.align_loss(fw["h_full"], fw["h_sparse"])
    O.attn_bwd(q, k, v, idx, cnt, w.block, w.sm_scale, grads["dh_full"][:1, :1],
               grads["dh_sparse"][:1, :1], 1.0, 1.0, n_total=inp["q"].numel(), rows=rows)
    dt = time.perf_counter() - t0
    blocksel = O.block_selection_matrix(idx, cnt)[0, 0]
    pf = int((rows + 1).sum())
    ps = 0
    for t in rows:
        i = t // w.block
        ps += int(blocksel[i, :i].sum()) * w.block + (t - i * w.block + 1)
    flops = 4 * w.D * pf + 10 * w.D * pf + 4 * w.D * ps
    return flops, dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, inp, grads, slices=8):
    """The oracle on a bounded sample: `slices` runs of query rows at the end
    of head (0, 0), about 8192 x 8192 row-key pairs in all at any T."""
    rows_per_slice = min(w.T, 8 * 1024 * 8192 // w.T) // slices
    flops = secs = 0.0
    for s in range(slices):
        hi = w.T - s * rows_per_slice
        f, t = oracle_slice(w, inp, grads, None, range(hi - rows_per_slice, hi))
        flops += f
        secs += t
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle", "seconds": round(secs, 2),
            "sample": f"fp64 numpy oracle, head (0,0) of {w.name}, query rows "
                      f"[{w.T - slices * rows_per_slice}, {w.T}): select + fwd + loss + bwd"}


def run_reference(args, world):
    w = workload(args)
    inp = make_inputs(w)
    grads = upstream_grads(w)
    rows = 512
    for _ in range(args.warmup):
        oracle_slice(w, inp, grads, None, range(w.T - rows, w.T))
    flops = secs = 0.0
    for _ in range(args.steps):
        f, t = oracle_slice(w, inp, grads, None, range(w.T - rows, w.T))
        flops += f
        secs += t
    value = flops / secs / 1e12
    cores = blas_threads()
    sample = (f"fp64 numpy oracle, head (0,0) of {w.name}, query rows [{w.T - rows}, {w.T}) "
              f"per step: select + fwd + loss + bwd")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": data_description(w),
        "config": workload_config(w, 1, "the oracle on one process's host cores"),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- distributed

def decode_bench(args, w, layer, stream, flush, dev):
    """One generation step at the last position of the workload (context T):
    the sparse stream over a key/value cache holding the step's K and V."""
    from block_sparse_full_b200 import ssa
    if w.D not in (64, 128) or w.topk > 64:
        return None
    cache = ssa.DecodeCache(layer.p, dev, layer.k.dtype)
    cache.k.copy_(layer.k)
    cache.v.copy_(layer.v)
    t = w.T - 1
    cache.pool_upto(t // w.block)
    q_t = layer.q[:, :, t].contiguous()
    # the step allocates nothing and never synchronises: a generation loop runs
    # it as a captured CUDA graph, which is what is timed (no host launch gaps)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        cache.step(t, q_t, idx=False)  # warm the allocator outside the capture
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        cache.step(t, q_t, idx=False)
    torch.cuda.synchronize(dev)
    ev = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        if i >= args.warmup:
            ev.append((e0, e1))
    torch.cuda.synchronize(dev)
    ssa.device_status()
    ms = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
    esz = 2 if w.dtype == "bf16" else 4
    i = t // w.block
    # keys and values of the selected blocks, the pooled-key scan, q and h
    per_head = w.topk * w.block * w.D * esz * 2 + i * w.D * 8 + 2 * w.D * esz
    nbytes = per_head * w.B * w.H
    del graph
    return {"kernels": ["decode_step_kernel"],
            "timed_as": "CUDA graph replay", "context": w.T, "ms": round(ms, 4), "hbm_bytes": nbytes,
            "hbm_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}


# The pages' one speed claim: at a 128k context SSA's inference (the sparse
# stream alone, MoBA's operations) runs about twice as fast as full attention
# ("Sintesi Tecnica: SSA", section 4, "Efficienza").  Placed on this library's
# own kernels: the sparse-only forward against the dual forward on the same
# selection and against the dual forward with every causal block selected
# (whose cost is that of one full-attention pass).
LONG_CONTEXT = Workload("bf16_T131072_H8_sink", B=1, H=8, T=131072, D=128, block=128, topk=16,
                        dtype="bf16", plant="sink", seed=6)


def long_context_bench(args, stream, flush, dev, w=LONG_CONTEXT, reps=3):
    from block_sparse_full_b200 import ssa
    inp = make_inputs(w)
    q, k, v = (inp[n].to(dev) for n in "qkv")
    del inp
    n = w.n_blocks
    p_k = ssa.params_for(q, w.block, w.topk, w.sm_scale)
    p_all = ssa.params_for(q, w.block, n, w.sm_scale)
    sel_k = ssa.select_blocks(p_k, q, k)
    sel_all = ssa.select_blocks(p_all, q, k)
    p_full, p_sel = pair_counts(w, sel_k[0].cpu().numpy(), sel_k[1].cpu().numpy())
    out = {}
    runs = {
        "sparse_only_k16": lambda: ssa.attn_fwd_sparse(p_k, q, k, v, sel_k[2], out=out.get("s")),
        "dual_k16": lambda: ssa.attn_fwd_dual(p_k, q, k, v, sel_k[2], out=out.get("d")),
        "dual_all_blocks": lambda: ssa.attn_fwd_dual(p_all, q, k, v, sel_all[2], out=out.get("d")),
    }
    out["s"] = runs["sparse_only_k16"]()
    out["d"] = runs["dual_k16"]()
    ms = {}
    for name, fn in runs.items():
        ev = []
        for i in range(1 + reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if i >= 1:
                ev.append((e0, e1))
        torch.cuda.synchronize(dev)
        ssa.device_status()
        ms[name] = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
    f_full = 4 * w.D * p_full * w.B * w.H
    f_sel = 4 * w.D * p_sel * w.B * w.H
    return {
        "workload": f"{w.name} (B{w.B} H{w.H} T{w.T} d{w.D} block {w.block} top-k {w.topk})",
        "ms": {k2: round(v2, 3) for k2, v2 in ms.items()},
        "tflops": {"sparse_only_k16": round(f_sel / (ms["sparse_only_k16"] * 1e-3) / 1e12, 1),
                   "dual_k16": round(f_full / (ms["dual_k16"] * 1e-3) / 1e12, 1),
                   "dual_all_blocks": round(f_full / (ms["dual_all_blocks"] * 1e-3) / 1e12, 1)},
        "speedup_sparse_vs_full_attention": round(ms["dual_all_blocks"] / ms["sparse_only_k16"], 2),
        "speedup_sparse_vs_dual": round(ms["dual_k16"] / ms["sparse_only_k16"], 2),
        "pages_claim": "about 2x over full attention at 128k (no hardware stated)",
        "reps": reps,
    }


def workload(args):
    """The named workload, with the selection budget overridden by --topk."""
    w = WORKLOADS[args.workload]
    if args.topk is None or args.topk == w.topk:
        return w
    if args.topk not in (getattr(w, "sweep", None) or ()):
        raise SystemExit(f"--topk {args.topk}: {w.name} sweeps {getattr(w, 'sweep', None)}")
    return dataclasses.replace(w, topk=args.topk, name=f"{w.name}_k{args.topk}")


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def reduce_max(x, world, dev):
    """Max of a per-rank value over all ranks (device time: the slowest rank)."""
    if world == 1:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def roofline_peak(timed_ms, burst, sustained):
    """(peak, kind) for a tensor-bound kernel timed inside a region of
    ``timed_ms``: the measured burst bf16 figure (best of a few GEMMs, clocks
    still at their maximum) for regions under a second, the sustained one
    (seconds of back-to-back GEMMs under the power cap) for longer ones."""
    if timed_ms < 1000.0:
        return burst, "burst (timed region under 1 s)"
    return sustained, "sustained (timed region of 1 s or more)"


def whole_job_tflops(flops_per_rank_step, world, max_ms_per_step):
    """Throughput of the whole job: every rank processes its own copy of the
    workload, so units scale with the rank count; time is the slowest rank's."""
    return flops_per_rank_step * world / (max_ms_per_step * 1e-3) / 1e12


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-long-context", dest="long_context", action="store_false",
                    help="skip the T=131072 inference comparison")
    ap.add_argument("--topk", type=int, default=None,
                    help="selection budget override (one of the workload's sweep values)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} but the launch has {world} rank(s): run N > 1 under "
                 "torch.distributed.run with --nproc-per-node N")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return 0
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120),
                                             device_id=dev)
    peaks, src = load_peaks()
    out = run_ours(args, rank, world, dev, peaks, src)
    if rank == 0:
        if world == 1 and args.cpu_baseline:
            w = workload(args)
            out["cpu_baseline"] = cpu_baseline(w, make_inputs(w), upstream_grads(w))
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
