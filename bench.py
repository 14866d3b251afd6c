#!/usr/bin/env python
"""Benchmark: one FP8 linear layer's training GEMMs on B200 through libfp8q.

Workload (one "step"): the DeepSeek-V3 expert-FFN up-projection linear layer with 4096 tokens,
C_in = 7168, C_out = 2048, bf16 operands resident in HBM:
    X to 1x128 + 128x1^T and W to 128x128, one launch -> Fprop Y = X W^T (bf16 [4096, 2048])
    dY to 1x128 + 128x1^T, one launch                 -> Dgrad dX = dY W  (bf16 [4096, 7168])
                                                         Wgrad dW = dY^T X (fp32 [2048, 7168])
5 kernel launches (8 with --separate-quant, which quantises each form of each tensor in its own
launch).  value = GEMM FLOPs (3 x 2*4096*2048*7168) / device time of the step.
L2 is flushed between steps, outside the timed step: a 256 MiB write, then a 256 MiB read of another
buffer, so each step starts with a cold L2 that holds no dirty lines of the flush itself.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of the step
(weak scaling, no data-path collective); the step time is the max over ranks.
--impl reference times the CPU oracle on a bounded slice of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

T_TOK, C_IN, C_OUT = 4096, 7168, 2048
MLA_WIDTHS = (1536, 512)                         # MLA query / KV compression widths
GEMM_FLOP = 2.0 * T_TOK * C_OUT * C_IN           # each of Fprop, Dgrad, Wgrad
STEP_FLOP = 3.0 * GEMM_FLOP
METRIC = ("block-scaled FP8 GEMM TFLOP/s (% dense FP8 peak); quantizer GB/s (% HBM)")
WORKLOAD = ("FP8 linear layer training GEMMs (act 1x128 + 128x1-transposed of X and of dY, "
            "weight 128x128, Fprop, Dgrad, Wgrad), tokens 4096, C_in 7168, C_out 2048")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0                              # nominal dense ratio (4.5 / 2.25 PFLOP/s)

# Algorithmic bytes per element: bf16 read (2) + code write (1) + one fp32 scale per group.
QB_1x128 = 2 + 1 + 4 / 128
QB_128x128 = 2 + 1 + 4 / (128 * 128)
QB_DUAL = 2 + 2 * (1 + 4 / 128)                  # one read, both code sets and scale sets


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's x (all ranks call it, in the same order); x itself on one rank."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


GEMM_SOURCES = ("fp8q.cu", "gemm.cuh", "ptx.cuh")   # the GEMM kernel and its schedule choice


def code_only(text: str) -> str:
    """C/C++ source without its comments, trailing blanks and blank lines (string literals that
    contain comment markers do not occur in the hashed files)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_hash(names=GEMM_SOURCES) -> str:
    """Hash of the GEMM sources' code (comments excluded): the DRAM counters in
    profiles/traffic.json describe the kernel built from exactly this code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_fine_grained_fp8q_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(code_only(f.read()).encode())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was taken on the GEMM
    sources as they are now (else None: the counters describe another kernel)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_hash") != source_hash():
        return None
    return d


# ------------------------------------------------------------------------------------------ #
# Clock sampling (read-only NVML queries)
# ------------------------------------------------------------------------------------------ #
class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.0):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        # The SM clock on every pass, the event reasons on every fourth: one NVML query takes
        # 0.1-0.2 ms, and a timed step lasts ~0.3 ms, so the clock gets a sample (or more) per step.
        nv = self._nvml
        n = 0
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                if n % 4 == 0:
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    for bit, name in self.REASONS.items():
                        if mask & bit and bit != 0x1:
                            self.reasons.add(name)
            except Exception:
                pass
            n += 1
            if self.period > 0:
                time.sleep(self.period)

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def summary(self, steps: int | None = None):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        out = {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
               "sm_mhz_min": float(min(self.samples)), "reasons": sorted(self.reasons),
               "samples": len(self.samples)}
        if steps:
            out["samples_per_step"] = round(len(self.samples) / steps, 2)
        return out


# ------------------------------------------------------------------------------------------ #
# GPU arm
# ------------------------------------------------------------------------------------------ #
OPS_FUSED = ["quant_forward_XW", "gemm_fprop", "act_dual_dY", "gemm_dgrad", "gemm_wgrad"]
OPS_SEPARATE = ["act_1x128_X", "weight_128x128_W", "gemm_fprop", "act_1x128_dY", "gemm_dgrad",
                "act_128x1t_X", "act_128x1t_dY", "gemm_wgrad"]


def make_buffers(torch, dev):
    from fp8_fine_grained_fp8q_b200 import synth
    d = synth.linear_layer(T_TOK, C_IN, C_OUT)
    host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory()
            for k, v in d.items()}
    t = {k: v.to(dev, non_blocking=False) for k, v in host.items()}
    u8, f32, bf16 = torch.uint8, torch.float32, torch.bfloat16
    e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)  # noqa: E731
    b = {
        "Xq": e((T_TOK, C_IN), u8), "sX": e((C_IN // 128, T_TOK), f32),
        "Wq": e((C_OUT, C_IN), u8), "sW": e((C_OUT // 128, C_IN // 128), f32),
        "Y": e((T_TOK, C_OUT), bf16),
        "dYq": e((T_TOK, C_OUT), u8), "sdY": e((C_OUT // 128, T_TOK), f32),
        "dX": e((T_TOK, C_IN), bf16),
        "Xtq": e((C_IN, T_TOK), u8), "sXt": e((T_TOK // 128, C_IN), f32),
        "dYtq": e((C_OUT, T_TOK), u8), "sdYt": e((T_TOK // 128, C_OUT), f32),
        "dW": e((C_OUT, C_IN), f32),
    }
    return host, t, b


def gemm_launches(ops, b):
    """The linear layer's three GEMM launches on the step's buffers."""
    return {
        "gemm_fprop": lambda: ops.gemm_blockscaled(ops.FPROP, b["Xq"], b["sX"], b["Wq"], b["sW"], b["Y"]),
        "gemm_dgrad": lambda: ops.gemm_blockscaled(ops.DGRAD, b["dYq"], b["sdY"], b["Wq"], b["sW"], b["dX"]),
        "gemm_wgrad": lambda: ops.gemm_blockscaled(ops.WGRAD, b["dYtq"], b["sdYt"], b["Xtq"], b["sXt"], b["dW"]),
    }


def step_ops(ops, t, b, separate=False):
    """The step as (names, zero-argument launches), all on torch's current stream.  By default
    X and dY are quantised to both forms in one pass each (act_dual); separate=True runs the
    1x128 and 128x1-transposed quantisers as their own launches."""
    gemms = gemm_launches(ops, b)
    quant = {
        "quant_forward_XW": lambda: ops.quant_forward(t["X"], t["W"], b["Xq"], b["sX"], b["Xtq"], b["sXt"],
                                                      b["Wq"], b["sW"]),
        "act_dual_X": lambda: ops.act_dual(t["X"], b["Xq"], b["sX"], b["Xtq"], b["sXt"]),
        "act_dual_dY": lambda: ops.act_dual(t["dY"], b["dYq"], b["sdY"], b["dYtq"], b["sdYt"]),
        "act_1x128_X": lambda: ops.act_1x128(t["X"], b["Xq"], b["sX"]),
        "act_1x128_dY": lambda: ops.act_1x128(t["dY"], b["dYq"], b["sdY"]),
        "act_128x1t_X": lambda: ops.act_128x1_transposed(t["X"], b["Xtq"], b["sXt"]),
        "act_128x1t_dY": lambda: ops.act_128x1_transposed(t["dY"], b["dYtq"], b["sdYt"]),
        "weight_128x128_W": lambda: ops.weight_128x128(t["W"], b["Wq"], b["sW"]),
    }
    names = OPS_SEPARATE if separate else OPS_FUSED
    table = {**gemms, **quant}
    return names, [table[n] for n in names]


def op_work():
    """Algorithmic work per launch: ('flop', F) or ('bytes', B)."""
    return {
        "quant_forward_XW": ("bytes", T_TOK * C_IN * QB_DUAL + C_OUT * C_IN * QB_128x128),
        "act_dual_X": ("bytes", T_TOK * C_IN * QB_DUAL),
        "act_dual_dY": ("bytes", T_TOK * C_OUT * QB_DUAL),
        "act_1x128_X": ("bytes", T_TOK * C_IN * QB_1x128),
        "weight_128x128_W": ("bytes", C_OUT * C_IN * QB_128x128),
        "gemm_fprop": ("flop", GEMM_FLOP),
        "act_1x128_dY": ("bytes", T_TOK * C_OUT * QB_1x128),
        "gemm_dgrad": ("flop", GEMM_FLOP),
        "act_128x1t_X": ("bytes", T_TOK * C_IN * QB_1x128),
        "act_128x1t_dY": ("bytes", T_TOK * C_OUT * QB_1x128),
        "gemm_wgrad": ("flop", GEMM_FLOP),
    }


def run_ue8m0_variant(ops, torch, t, b, flush_l2, steps):
    """Not the headline: the same five-launch step with power-of-two (UE8M0) scales, whose GEMMs
    run on the block-scaled tensor-core MMA without per-128-K promotion (a separate mode, not the
    pages' method).  Whole steps with an event on each side, then each launch alone."""
    launches = {
        "quant_forward_XW": lambda: ops.quant_forward(t["X"], t["W"], b["Xq"], b["sX"], b["Xtq"], b["sXt"],
                                                      b["Wq"], b["sW"], scale_fmt="ue8m0"),
        "gemm_fprop": lambda: ops.gemm_blockscaled_ue8m0(ops.FPROP, b["Xq"], b["sX"], b["Wq"], b["sW"], b["Y"]),
        "act_dual_dY": lambda: ops.act_dual(t["dY"], b["dYq"], b["sdY"], b["dYtq"], b["sdYt"], scale_fmt="ue8m0"),
        "gemm_dgrad": lambda: ops.gemm_blockscaled_ue8m0(ops.DGRAD, b["dYq"], b["sdY"], b["Wq"], b["sW"], b["dX"]),
        "gemm_wgrad": lambda: ops.gemm_blockscaled_ue8m0(ops.WGRAD, b["dYtq"], b["sdYt"], b["Xtq"], b["sXt"], b["dW"]),
    }
    fs = list(launches.values())
    for _ in range(3):
        flush_l2()
        for f in fs:
            f()
    n = max(5, min(steps, 30))
    step_ms, per = [], {k: [] for k in launches}
    for _ in range(n):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for f in fs:
            f()
        e1.record()
        torch.cuda.synchronize()
        step_ms.append(e0.elapsed_time(e1))
    for _ in range(n):
        flush_l2()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(fs) + 1)]
        evs[0].record()
        for i, f in enumerate(fs):
            f()
            evs[i + 1].record()
        torch.cuda.synchronize()
        for i, k in enumerate(launches):
            per[k].append(evs[i].elapsed_time(evs[i + 1]))
    status = ops.device_status()
    if status != ops.DEV_OK:
        raise RuntimeError(f"device status {status} in the UE8M0 variant")
    ms = statistics.median(step_ms)
    kern = {k: round(statistics.median(v), 5) for k, v in per.items()}
    return {"step_ms": round(ms, 5), "step_TFLOP/s": round(STEP_FLOP / (ms * 1e-3) / 1e12, 1),
            "kernels_ms": kern,
            "gemm_TFLOP/s": {k: round(GEMM_FLOP / (kern[k] * 1e-3) / 1e12, 1)
                             for k in ("gemm_fprop", "gemm_dgrad", "gemm_wgrad")},
            "steps": n, "scales": "power of two (UE8M0); tcgen05.mma kind::mxf8f6f4, whole-K TMEM accumulation"}


def run_ours(args, rank, world, dist):
    import torch
    from fp8_fine_grained_fp8q_b200 import ops

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ops.lib()                                      # fail loudly if the library is missing
    host, t, b = make_buffers(torch, dev)
    OPS, launches = step_ops(ops, t, b, separate=args.separate_quant)
    gemm_launch = gemm_launches(ops, b)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        # The write evicts everything the last step left in L2; reading a second buffer then
        # writes the flush's own dirty lines back, outside the step.
        flush_w.zero_()
        flush_r.sum()
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush_l2()
        for f in launches:
            f()
    torch.cuda.synchronize()
    status = ops.device_status(dev)
    if status != ops.DEV_OK:
        raise RuntimeError(f"device status {status} after warm-up")

    # Timed region: each step bracketed by two events only (an event between two launches would
    # serialise them and hide the launch overlap the kernels are built for).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        start.record()
        for s in range(args.steps):
            flush_l2()
            evs[s][0].record()
            for f in launches:
                f()
            evs[s][1].record()
        end.record()
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    status = ops.device_status(dev)
    if status != ops.DEV_OK:
        raise RuntimeError(f"device status {status} in the timed region")
    step_ms = [evs[s][0].elapsed_time(evs[s][1]) for s in range(args.steps)]

    # Per-kernel breakdown, outside the timed region: the same steps with an event after every
    # launch (each kernel then runs alone, so these times include its full launch and tail).
    n_ev = len(launches) + 1
    bsteps = min(args.steps, 20)
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(bsteps)]
    for s in range(bsteps):
        flush_l2()
        bevs[s][0].record()
        for i, f in enumerate(launches):
            f()
            bevs[s][i + 1].record()
    torch.cuda.synchronize()
    per_op = {name: [] for name in OPS}
    for s in range(bsteps):
        for i, name in enumerate(OPS):
            per_op[name].append(bevs[s][i].elapsed_time(bevs[s][i + 1]))

    # Not part of the step: Fprop with the next layer's 1x128 quantisation of Y fused into its
    # epilogue, against Fprop followed by the separate quantiser.
    yq = torch.empty((T_TOK, C_OUT), dtype=torch.uint8, device=dev)
    ys = torch.empty((C_OUT // 128, T_TOK), dtype=torch.float32, device=dev)
    fused_runs = {
        "fprop": lambda: ops.gemm_blockscaled(ops.FPROP, b["Xq"], b["sX"], b["Wq"], b["sW"], b["Y"]),
        "fprop_then_act_1x128_Y": lambda: (ops.gemm_blockscaled(ops.FPROP, b["Xq"], b["sX"], b["Wq"], b["sW"], b["Y"]),
                                           ops.act_1x128(b["Y"], yq, ys)),
        "fprop_fused_quant_Y": lambda: ops.gemm_blockscaled_quant(ops.FPROP, b["Xq"], b["sX"], b["Wq"], b["sW"],
                                                                  b["Y"], yq, ys),
    }
    fused_ms = {}
    for name, f in fused_runs.items():
        ts = []
        for _ in range(10):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        fused_ms[name] = round(statistics.median(ts[2:]), 5)
    # Not part of the step either: the MLA-shaped Fprop GEMMs (query / KV down-projections,
    # X [4096, 7168] times W [1536 | 512, 7168]^T), on the step's quantised X and their own
    # seeded weights quantised 128x128 on the device.
    mla, mla_ops = {}, {}
    for n_mla in MLA_WIDTHS:
        from fp8_fine_grained_fp8q_b200 import synth
        wm = torch.from_numpy(synth.weights(n_mla, C_IN, seed=synth.SEED_BASE + 3 + n_mla).view(np.int16)).view(
            torch.bfloat16).to(dev)
        wq, ws, _ = ops.weight_128x128(wm)
        ym = torch.empty((T_TOK, n_mla), dtype=torch.bfloat16, device=dev)
        f = lambda: ops.gemm_blockscaled(ops.FPROP, b["Xq"], b["sX"], wq, ws, ym)  # noqa: E731
        for _ in range(3):
            f()
        ts = []
        for _ in range(20):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        mla[n_mla] = statistics.median(ts)
        mla_ops[n_mla] = (wq, ws, ym)
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status after the MLA-shaped GEMMs")

    # Each GEMM under the conditions it meets inside the step: its operands were just written (so
    # they sit in L2) and it is launched right behind another kernel (programmatic dependent launch
    # overlaps the two).  After an L2 flush one launch brings the operands back; then 10 launches
    # back to back between two events; median of 7 such runs.  The per-launch breakdown above puts
    # an event between launches instead, which serialises them and adds the launch latency to
    # each kernel's time.
    in_step_runs = {
        "gemm_fprop": (gemm_launch["gemm_fprop"], GEMM_FLOP),
        "gemm_dgrad": (gemm_launch["gemm_dgrad"], GEMM_FLOP),
        "gemm_wgrad": (gemm_launch["gemm_wgrad"], GEMM_FLOP),
    }
    for n_mla, (wq, ws, ym) in mla_ops.items():
        in_step_runs[f"gemm_fprop_mla_n{n_mla}"] = (
            (lambda wq=wq, ws=ws, ym=ym: ops.gemm_blockscaled(ops.FPROP, b["Xq"], b["sX"], wq, ws, ym)),
            2.0 * T_TOK * n_mla * C_IN)
    in_step = {}
    for name, (f, flop) in in_step_runs.items():
        for _ in range(3):
            f()
        reps = []
        for _ in range(7):
            flush_l2()
            f()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(10):
                f()
            e1.record()
            torch.cuda.synchronize()
            reps.append(e0.elapsed_time(e1) / 10)
        in_step[name] = (statistics.median(reps), flop)
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status after the in-step GEMM runs")

    # The quantisers' device time without the launch gap, still reading HBM: 12 launches back to
    # back between two events, each on its own copy of the inputs (3 copies of X, 6 of W, 8 of
    # dY: between two uses of a copy at least 170 MB pass through the 126 MB L2), median of 7.
    xs = [t["X"]] + [t["X"].clone() for _ in range(2)]
    wsx = [t["W"]] + [t["W"].clone() for _ in range(5)]
    dys = [t["dY"]] + [t["dY"].clone() for _ in range(7)]
    q_runs = {
        "quant_forward_XW": lambda i: ops.quant_forward(xs[i % 3], wsx[i % 3], b["Xq"], b["sX"], b["Xtq"], b["sXt"],
                                                        b["Wq"], b["sW"]),
        "act_dual_dY": lambda i: ops.act_dual(dys[i % 8], b["dYq"], b["sdY"], b["dYtq"], b["sdYt"]),
        # the single-form quantisers (not in the step, which uses the fused ones above)
        "act_1x128_X": lambda i: ops.act_1x128(xs[i % 3], b["Xq"], b["sX"]),
        "act_128x1t_X": lambda i: ops.act_128x1_transposed(xs[i % 3], b["Xtq"], b["sXt"]),
        "weight_128x128_W": lambda i: ops.weight_128x128(wsx[i % 6], b["Wq"], b["sW"]),
    }
    q_dev = {}
    for name, f in q_runs.items():
        for i in range(8):
            f(i)
        reps = []
        for _ in range(7):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(12):
                f(i)
            e1.record()
            torch.cuda.synchronize()
            reps.append(e0.elapsed_time(e1) / 12)
        q_dev[name] = statistics.median(reps)
    del xs, wsx, dys
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status after the quantiser device-time runs")
    sum_step_ms = float(sum(step_ms))
    total_ms = start.elapsed_time(end)
    sum_step_ms = max_over_ranks(sum_step_ms, dist, dev)
    ms_per_step = sum_step_ms / args.steps
    value = world * STEP_FLOP / (ms_per_step * 1e-3) / 1e12

    # End to end through the same public calls, host buffers: H2D of this step's inputs from
    # pinned memory, the step, D2H of its outputs, all in the timed region.
    out_host = {k: torch.empty(b[k].shape, dtype=b[k].dtype, pin_memory=True)
                for k in ("Y", "dX", "dW")}
    e2e_steps = max(3, min(args.steps, 20))
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())
    e2e_ms = []
    for s in range(e2e_steps + 2):
        flush_l2()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for k in host:
            t[k].copy_(host[k], non_blocking=True)
        for f in launches:
            f()
        for k in out_host:
            out_host[k].copy_(b[k], non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        if s >= 2:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e_sum = float(sum(e2e_ms))
    e2e_sum = max_over_ranks(e2e_sum, dist, dev)
    e2e_value = world * STEP_FLOP / (e2e_sum / len(e2e_ms) * 1e-3) / 1e12

    ue8m0 = run_ue8m0_variant(ops, torch, t, b, flush_l2, args.steps)

    peaks, peak_kind = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    hbm = peaks["hbm_gbs"]
    work = op_work()
    kernels = {}
    for name in OPS:
        ms = statistics.mean(per_op[name])
        kind, amount = work[name]
        if kind == "flop":
            ach = amount / (ms * 1e-3) / 1e12
            kernels[name] = {"ms": round(ms, 5), "TFLOP/s": round(ach, 1),
                             "frac_fp8_peak": round(ach / fp8_peak, 4)}
        else:
            ach = amount / (ms * 1e-3) / 1e9
            kernels[name] = {"ms": round(ms, 5), "GB/s": round(ach, 1),
                             "frac_hbm": round(ach / hbm, 4)}
    for n_mla, ms in mla.items():
        flop = 2.0 * T_TOK * n_mla * C_IN
        ach = flop / (ms * 1e-3) / 1e12
        kernels[f"gemm_fprop_mla_n{n_mla}"] = {
            "ms": round(ms, 5), "TFLOP/s": round(ach, 1), "frac_fp8_peak": round(ach / fp8_peak, 4),
            "shape": f"{T_TOK}x{n_mla}x{C_IN}", "in_step": False}
    kernels_in_step = {}
    for name, (ms, flop) in in_step.items():
        ach = flop / (ms * 1e-3) / 1e12
        kernels_in_step[name] = {"ms": round(ms, 5), "TFLOP/s": round(ach, 1), "frac_fp8_peak": round(ach / fp8_peak, 4)}
    gemm_ms_serial = statistics.mean([statistics.mean(per_op[n]) for n in ("gemm_fprop", "gemm_dgrad", "gemm_wgrad")])
    gemm_ms = statistics.mean([in_step[n][0] for n in ("gemm_fprop", "gemm_dgrad", "gemm_wgrad")])
    gemm_ach = GEMM_FLOP / (gemm_ms * 1e-3) / 1e12
    traffic = load_traffic()
    roofline = {
        "kernel": "gemm_blockscaled_kernel (fprop, dgrad, wgrad launches; 120.26 GFLOP each)",
        "bound": "tensor", "achieved": round(gemm_ach, 1), "peak": round(fp8_peak, 1),
        "unit": "TFLOP/s", "frac": round(gemm_ach / fp8_peak, 4),
        "peak_source": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {FP8_OVER_BF16} "
                       "(nominal dense FP8/BF16 ratio)",
        "traffic": (traffic or {}).get("gemm_bytes_per_launch"),
        "duration": "mean over the three GEMMs of the per-launch time under in-step conditions (kernels_in_step)",
        "achieved_serialized": round(GEMM_FLOP / (gemm_ms_serial * 1e-3) / 1e12, 1),
    }
    q_ms = sum(statistics.mean(per_op[n]) for n in OPS if n.startswith(("act", "weight", "quant")))
    q_bytes = sum(work[n][1] for n in OPS if n.startswith(("act", "weight", "quant")))
    quantizers_device = {}
    for name, ms in q_dev.items():
        ach = work[name][1] / (ms * 1e-3) / 1e9
        quantizers_device[name] = {"ms": round(ms, 5), "GB/s": round(ach, 1), "frac_hbm": round(ach / hbm, 4)}
    step_q = ("quant_forward_XW", "act_dual_dY")
    qd_ms, qd_bytes = sum(q_dev[n] for n in step_q), sum(work[n][1] for n in step_q)
    quantizers_device["aggregate"] = {"GB/s": round(qd_bytes / (qd_ms * 1e-3) / 1e9, 1),
                                      "frac_hbm": round(qd_bytes / (qd_ms * 1e-3) / 1e9 / hbm, 4),
                                      "launches": list(step_q)}
    quantizers_device["method"] = ("12 launches back to back between two events, each on its own copy of the "
                                   "inputs (no copy is in L2 when it is read), median of 7: device time "
                                   "without the launch gap that `kernels` carries; the aggregate is the "
                                   "step's two quantiser launches")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3 (fp32 accumulate)", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "tokens": T_TOK, "c_in": C_IN, "c_out": C_OUT,
                   "l2": "flushed before every step, outside the step: 256 MiB write, then 256 MiB read of another buffer",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roofline,
        "quantizers": {"GB/s": quantizers_device["aggregate"]["GB/s"],
                       "frac_hbm": quantizers_device["aggregate"]["frac_hbm"],
                       "hbm_peak_gbs": hbm, "peak_source": peak_kind,
                       "method": "the step's quantiser launches, device time (quantizers_device)",
                       "serialized": {"GB/s": round(q_bytes / (q_ms * 1e-3) / 1e9, 1),
                                      "frac_hbm": round(q_bytes / (q_ms * 1e-3) / 1e9 / hbm, 4),
                                      "method": "events around each launch of a separate pass (kernels)"}},
        "quantizers_device": quantizers_device,
        "kernels": kernels,
        "kernels_method": "events after every launch of a separate pass of the step (serialised launches)",
        "kernels_in_step": kernels_in_step,
        "fused_output_quant_ms": fused_ms,
        "ue8m0_variant": ue8m0,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": len(e2e_ms)},
        "gpu_launches": len(launches) * args.steps,
        "clocks": clocks.summary(args.steps),
        "wall_ms_timed_region": round(total_ms, 3),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
    return line


# ------------------------------------------------------------------------------------------ #
# CPU oracle (baseline leg and --impl reference)
# ------------------------------------------------------------------------------------------ #
SLICE_T, SLICE_OUT = 128, 128


def oracle_slice_inputs():
    from fp8_fine_grained_fp8q_b200 import synth
    d = synth.linear_layer(T_TOK, C_IN, C_OUT)
    return {"X": np.ascontiguousarray(d["X"][:SLICE_T]),
            "W": np.ascontiguousarray(d["W"][:SLICE_OUT]),
            "dY": np.ascontiguousarray(d["dY"][:SLICE_T, :SLICE_OUT])}


def oracle_step(oracle, d):
    xq, xs = oracle.quant_1x128(d["X"])
    wq, ws, _ = oracle.quant_128x128(d["W"])
    oracle.gemm(oracle.FPROP, xq, xs, wq, ws)
    gq, gs = oracle.quant_1x128(d["dY"])
    oracle.gemm(oracle.DGRAD, gq, gs, wq, ws)
    xtq, xts = oracle.quant_128x1_t(d["X"])
    gtq, gts = oracle.quant_128x1_t(d["dY"])
    oracle.gemm(oracle.WGRAD, gtq, gts, xtq, xts)


SLICE_FLOP = 3 * 2.0 * SLICE_T * SLICE_OUT * C_IN
SLICE_DESC = (f"the same step on a slice of the same layer: {SLICE_T} of 4096 tokens and "
              f"{SLICE_OUT} of 2048 output channels, full C_in = 7168 (1/512 of the GEMM work); "
              "value = GEMM FLOPs of the slice / oracle time")


def cpu_baseline(budget_s: float = 15.0):
    import oracle
    d = oracle_slice_inputs()
    oracle_step(oracle, d)                         # warm (and build) once
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 2:
        t0 = time.perf_counter()
        oracle_step(oracle, d)
        times.append(time.perf_counter() - t0)
    mean = statistics.mean(times)
    return {"value": round(SLICE_FLOP / mean / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": SLICE_DESC + f"; {len(times)} repetitions, {sum(times):.1f} s",
            "quantizers": cpu_quantizers(oracle)}


def cpu_quantizers(oracle, budget_s: float = 2.0):
    """The oracle's three quantisers on 512 tokens of X [., 7168] (both activation forms) and
    256 rows of W [., 7168], as algorithmic GB/s, on one thread and on all cores."""
    import ctypes
    from fp8_fine_grained_fp8q_b200 import synth
    d = synth.linear_layer(T_TOK, C_IN, C_OUT)
    x, w = np.ascontiguousarray(d["X"][:512]), np.ascontiguousarray(d["W"][:256])
    nbytes = 2 * x.size * QB_1x128 + w.size * QB_128x128

    def run():
        oracle.quant_1x128(x)
        oracle.quant_128x1_t(x)
        oracle.quant_128x128(w)

    def rate():
        run()
        n, t0 = 0, time.perf_counter()
        while n < 2 or time.perf_counter() - t0 < budget_s:
            run()
            n += 1
        return nbytes * n / (time.perf_counter() - t0) / 1e9

    out = {"unit": "GB/s", "sample": "X [512, 7168] to 1x128 and 128x1-transposed, W [256, 7168] to 128x128 "
                                     f"({nbytes / 1e6:.1f} MB of algorithmic traffic per pass)"}
    cores = oracle.num_threads()
    out["all_cores"], out["cores"] = round(rate(), 3), cores
    out["one_thread"] = None
    try:
        gomp = ctypes.CDLL("libgomp.so.1")      # the OpenMP runtime the oracle's library runs on
    except OSError:
        return out
    gomp.omp_set_num_threads(1)
    try:
        if oracle.num_threads() == 1:
            out["one_thread"] = round(rate(), 3)
    finally:
        gomp.omp_set_num_threads(cores)
    return out


def run_reference(args, rank, world):
    import oracle
    d = oracle_slice_inputs()
    for _ in range(args.warmup):
        oracle_step(oracle, d)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(oracle, d)
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    value = SLICE_FLOP / (ms * 1e-3) / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "tokens": T_TOK, "c_in": C_IN, "c_out": C_OUT,
                   "sample": SLICE_DESC},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": SLICE_DESC},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------------------ #
# Secondary workload: the grouped MoE Fprop (--workload moe)
# ------------------------------------------------------------------------------------------ #
MOE_TOKENS, MOE_E, MOE_TOPK, MOE_N, MOE_K = 8192, 256, 8, 2048, 7168
MOE_WORKLOAD = ("grouped MoE Fprop: 8192 tokens x top-8 of 256 experts (Zipf(1.1)-skewed, 8 empty), "
                "act 1x128 of the expert-ordered rows [65536, 7168] + weight 128x128 of all experts "
                "[256 x 2048, 7168] + ragged grouped GEMM")


def run_moe(args, rank, world, dist):
    """One step = 1x128 quantisation of the expert-ordered activations, 128x128 quantisation of all
    expert weights, and the grouped GEMM; value = grouped-GEMM FLOPs / step time.  Inputs are
    generated on the device (seeded): X ~ N(0,1) with 7 outlier channels x100, W_e ~ N(0, 0.02)."""
    import torch
    from fp8_fine_grained_fp8q_b200 import ops, synth

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ops.lib()
    expert_of, counts = synth.moe_routing(tokens=MOE_TOKENS, experts=MOE_E, top_k=MOE_TOPK)
    token_idx, off = synth.moe_grouped_rows(expert_of, MOE_E)
    mtot = int(off[-1])
    g = torch.Generator(device=dev)
    g.manual_seed(synth.SEED_BASE + 5)
    x = torch.randn((MOE_TOKENS, MOE_K), device=dev, generator=g)
    outl = torch.randperm(MOE_K, device=dev, generator=g)[: round(0.001 * MOE_K)]
    x[:, outl] *= 100.0
    xg = x.to(torch.bfloat16)[torch.from_numpy(token_idx).to(dev)].contiguous()
    del x
    w = torch.empty((MOE_E * MOE_N, MOE_K), dtype=torch.bfloat16, device=dev)
    for e0 in range(0, MOE_E, 32):
        w[e0 * MOE_N:(e0 + 32) * MOE_N] = (0.02 * torch.randn((32 * MOE_N, MOE_K), device=dev, generator=g)).to(torch.bfloat16)
    offsets = torch.from_numpy(off).to(dev)
    xq = torch.empty((mtot, MOE_K), dtype=torch.uint8, device=dev)
    sx = torch.empty((MOE_K // 128, mtot), dtype=torch.float32, device=dev)
    wq = torch.empty((MOE_E * MOE_N, MOE_K), dtype=torch.uint8, device=dev)
    sw = torch.empty((MOE_E * MOE_N // 128, MOE_K // 128), dtype=torch.float32, device=dev)
    out = torch.empty((mtot, MOE_N), dtype=torch.bfloat16, device=dev)
    names = ["act_1x128_X", "weight_128x128_W", "grouped_gemm"]
    launches = [
        lambda: ops.act_1x128(xg, xq, sx),
        lambda: ops.weight_128x128(w, wq, sw),
        lambda: ops.grouped_gemm_blockscaled(xq, sx, wq.view(MOE_E, MOE_N, MOE_K),
                                             sw.view(MOE_E, MOE_N // 128, MOE_K // 128), offsets, out),
    ]
    flop = 2.0 * mtot * MOE_N * MOE_K
    work = {"act_1x128_X": ("bytes", mtot * MOE_K * QB_1x128),
            "weight_128x128_W": ("bytes", MOE_E * MOE_N * MOE_K * QB_128x128),
            "grouped_gemm": ("flop", flop)}
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.sum()

    for _ in range(args.warmup):
        flush_l2()
        for f in launches:
            f()
    torch.cuda.synchronize()
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        for s_ in range(args.steps):
            flush_l2()
            evs[s_][0].record()
            for f in launches:
                f()
            evs[s_][1].record()
        torch.cuda.synchronize()
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status in the timed region")
    ms_per_step = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)
    bsteps = min(args.steps, 10)
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(launches) + 1)] for _ in range(bsteps)]
    for s_ in range(bsteps):
        flush_l2()
        bevs[s_][0].record()
        for i, f in enumerate(launches):
            f()
            bevs[s_][i + 1].record()
    torch.cuda.synchronize()
    # Not part of the step: the experts' input gradient, grouped Dgrad dX = dY W_e over the same
    # rows, with the same (forward) expert weights and a seeded dY quantised on the device.
    dy = (1e-3 * torch.randn((mtot, MOE_N), device=dev, generator=g)).to(torch.bfloat16)
    dyq = torch.empty((mtot, MOE_N), dtype=torch.uint8, device=dev)
    dys = torch.empty((MOE_N // 128, mtot), dtype=torch.float32, device=dev)
    ops.act_1x128(dy, dyq, dys)
    dx = torch.empty((mtot, MOE_K), dtype=torch.bfloat16, device=dev)
    dts = []
    for _ in range(8):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ops.grouped_gemm_blockscaled_dgrad(dyq, dys, wq.view(MOE_E, MOE_N, MOE_K),
                                           sw.view(MOE_E, MOE_N // 128, MOE_K // 128), offsets, dx)
        e1.record()
        torch.cuda.synchronize()
        dts.append(e0.elapsed_time(e1))
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status after the grouped Dgrad")
    dgrad_ms = statistics.median(dts[2:])
    # Not part of the step either: the experts' weight gradients, dW_e = dY_e^T X_e over each
    # expert's own tokens (ragged 128x1 quantisation of dY and X, then the K-grouped GEMM).
    dw = torch.empty((MOE_E, MOE_N, MOE_K), dtype=torch.float32, device=dev)
    kcap = ops.ragged_capacity(mtot, MOE_E)
    dyt = torch.empty((MOE_N, kcap), dtype=torch.uint8, device=dev)
    sdyt = torch.empty((kcap // 128, MOE_N), dtype=torch.float32, device=dev)
    xt = torch.empty((MOE_K, kcap), dtype=torch.uint8, device=dev)
    sxt = torch.empty((kcap // 128, MOE_K), dtype=torch.float32, device=dev)
    wts, qts = [], []
    for _ in range(6):
        flush_l2()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        ops.act_128x1_transposed_ragged(dy, offsets, kcap, dyt, sdyt)
        ops.act_128x1_transposed_ragged(xg, offsets, kcap, xt, sxt)
        e1.record()
        ops.grouped_gemm_blockscaled_wgrad(dyt, sdyt, xt, sxt, offsets, mtot, dw)
        e2.record()
        torch.cuda.synchronize()
        qts.append(e0.elapsed_time(e1))
        wts.append(e1.elapsed_time(e2))
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status after the grouped Wgrad")
    del dw
    wgrad_ms, rq_ms = statistics.median(wts[2:]), statistics.median(qts[2:])
    rq_bytes = mtot * (MOE_N + MOE_K) * QB_1x128
    peaks, peak_kind = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    kernels = {}
    for i, name in enumerate(names):
        ms = statistics.mean(b[i].elapsed_time(b[i + 1]) for b in bevs)
        kind, amount = work[name]
        if kind == "flop":
            ach = amount / (ms * 1e-3) / 1e12
            kernels[name] = {"ms": round(ms, 4), "TFLOP/s": round(ach, 1), "frac_fp8_peak": round(ach / fp8_peak, 4)}
        else:
            ach = amount / (ms * 1e-3) / 1e9
            kernels[name] = {"ms": round(ms, 4), "GB/s": round(ach, 1), "frac_hbm": round(ach / peaks["hbm_gbs"], 4)}
    g_ms = kernels["grouped_gemm"]["ms"]
    # The grouped GEMM's algorithmic bytes: A codes + scales, the weights (codes + scales) of the
    # experts that hold rows (an empty expert's weights are never read), the bf16 output.
    live = int((counts > 0).sum())
    g_bytes = (mtot * MOE_K * (1 + 4 / 128) + live * MOE_N * MOE_K * (1 + 4 / (128 * 128))
               + mtot * MOE_N * 2)
    g_gbs = g_bytes / (g_ms * 1e-3) / 1e9
    g_tf = flop / (g_ms * 1e-3) / 1e12
    # Roofline bound: whichever of the two floors is the longer one at these sizes.
    t_hbm, t_tensor = g_bytes / (peaks["hbm_gbs"] * 1e9), flop / (fp8_peak * 1e12)
    trf = load_traffic()
    g_traffic = trf.get("moe_grouped_bytes_per_launch") if trf else None
    if t_hbm >= t_tensor:
        roof = {"kernel": "gemm_blockscaled_kernel (grouped)", "bound": "hbm", "achieved": round(g_gbs, 1),
                "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s", "frac": round(g_gbs / peaks["hbm_gbs"], 4),
                "peak_source": peak_kind, "traffic": g_traffic, "algorithmic_bytes": int(g_bytes),
                "tensor": {"achieved": round(g_tf, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                           "frac": round(g_tf / fp8_peak, 4)}}
    else:
        roof = {"kernel": "gemm_blockscaled_kernel (grouped)", "bound": "tensor", "achieved": round(g_tf, 1),
                "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(g_tf / fp8_peak, 4),
                "peak_source": f"{peak_kind} bf16 burst x {FP8_OVER_BF16}", "traffic": g_traffic,
                "algorithmic_bytes": int(g_bytes),
                "hbm": {"achieved": round(g_gbs, 1), "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
                        "frac": round(g_gbs / peaks["hbm_gbs"], 4)}}
    roof["floors_ms"] = {"hbm": round(t_hbm * 1e3, 4), "tensor": round(t_tensor * 1e3, 4)}
    return {
        "metric": METRIC, "value": round(world * flop / (ms_per_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3 (fp32 accumulate)", "data": "synthetic (seeded, generated on the device)",
        "config": {"workload": MOE_WORKLOAD, "rows": mtot, "experts": MOE_E,
                   "empty_experts": int((counts == 0).sum()), "max_rows": int(counts.max()),
                   "n": MOE_N, "k": MOE_K, "l2": "flushed before every step (256 MiB write, then read)"},
        "roofline": roof,
        "kernels": kernels,
        "grouped_dgrad": {"ms": round(dgrad_ms, 4), "TFLOP/s": round(flop / (dgrad_ms * 1e-3) / 1e12, 1),
                          "frac_fp8_peak": round(flop / (dgrad_ms * 1e-3) / 1e12 / fp8_peak, 4),
                          "note": "dX [rows, 7168] = dY [rows, 2048] W_e, not part of the step"},
        "grouped_wgrad": {"ms": round(wgrad_ms, 4), "TFLOP/s": round(flop / (wgrad_ms * 1e-3) / 1e12, 1),
                          "frac_fp8_peak": round(flop / (wgrad_ms * 1e-3) / 1e12 / fp8_peak, 4),
                          "dw_bytes": MOE_E * MOE_N * MOE_K * 4,
                          "note": "dW_e [2048, 7168] fp32 for all 256 experts (15 GB written), "
                                  "FLOPs counted over the real tokens; not part of the step"},
        "ragged_128x1_quant": {"ms": round(rq_ms, 4), "GB/s": round(rq_bytes / (rq_ms * 1e-3) / 1e9, 1),
                               "note": "dY and X of the expert rows to the grouped-Wgrad operand form"},
        "e2e": None,
        "e2e_note": "not measured for this secondary workload (the expert weights alone are 7.5 GB of H2D per step)",
        "gpu_launches": len(launches) * args.steps,
        "clocks": clocks.summary(),
    }


def profile_moe(experts: int):
    """One launch of the grouped MoE Fprop GEMM on the MoE workload's operands (8192 tokens x top-8
    routed over `experts` experts), after quantising them once, for a profiler capture:
    `-k regex:gemm_blockscaled -c 1` takes exactly that launch."""
    import torch
    from fp8_fine_grained_fp8q_b200 import ops, synth
    dev = torch.device("cuda", 0)
    expert_of, _ = synth.moe_routing(tokens=MOE_TOKENS, experts=experts, top_k=MOE_TOPK,
                                     n_empty=max(1, experts // 32))
    token_idx, off = synth.moe_grouped_rows(expert_of, experts)
    mtot = int(off[-1])
    g = torch.Generator(device=dev)
    g.manual_seed(synth.SEED_BASE + 5)
    x = torch.randn((MOE_TOKENS, MOE_K), device=dev, generator=g)
    x[:, torch.randperm(MOE_K, device=dev, generator=g)[: round(0.001 * MOE_K)]] *= 100.0
    xg = x.to(torch.bfloat16)[torch.from_numpy(token_idx).to(dev)].contiguous()
    del x
    wq = torch.empty((experts * MOE_N, MOE_K), dtype=torch.uint8, device=dev)
    sw = torch.empty((experts * MOE_N // 128, MOE_K // 128), dtype=torch.float32, device=dev)
    for e0 in range(0, experts, 32):
        n = min(32, experts - e0)
        w = (0.02 * torch.randn((n * MOE_N, MOE_K), device=dev, generator=g)).to(torch.bfloat16)
        ops.weight_128x128(w, wq[e0 * MOE_N:(e0 + n) * MOE_N], sw[e0 * MOE_N // 128:(e0 + n) * MOE_N // 128])
        del w
    xq, sx = ops.act_1x128(xg)
    out = torch.empty((mtot, MOE_N), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    ops.grouped_gemm_blockscaled(xq, sx, wq.view(experts, MOE_N, MOE_K), sw.view(experts, MOE_N // 128, MOE_K // 128),
                                 torch.from_numpy(off).to(dev), out)
    torch.cuda.synchronize()
    if ops.device_status(dev) != ops.DEV_OK:
        raise RuntimeError("device status after the grouped GEMM")
    print(json.dumps({"profile_moe": experts, "rows": mtot, "status": "ok"}))


def profile_gemms(fmt: str):
    """The linear layer's three GEMMs, one launch each, after one quantisation pass (for a profiler
    capture: `-k regex:gemm_blockscaled -c 3` takes exactly these launches)."""
    import torch
    from fp8_fine_grained_fp8q_b200 import ops
    dev = torch.device("cuda", 0)
    _, t, b = make_buffers(torch, dev)
    ops.quant_forward(t["X"], t["W"], b["Xq"], b["sX"], b["Xtq"], b["sXt"], b["Wq"], b["sW"], scale_fmt=fmt)
    ops.act_dual(t["dY"], b["dYq"], b["sdY"], b["dYtq"], b["sdYt"], scale_fmt=fmt)
    gemm = ops.gemm_blockscaled if fmt == "fp32" else ops.gemm_blockscaled_ue8m0
    torch.cuda.synchronize()
    gemm(ops.FPROP, b["Xq"], b["sX"], b["Wq"], b["sW"], b["Y"])
    gemm(ops.DGRAD, b["dYq"], b["sdY"], b["Wq"], b["sW"], b["dX"])
    gemm(ops.WGRAD, b["dYtq"], b["sdYt"], b["Xtq"], b["sXt"], b["dW"])
    torch.cuda.synchronize()
    status = ops.device_status(dev)
    if status != ops.DEV_OK:
        raise RuntimeError(f"device status {status}")
    print(json.dumps({"profile_gemms": fmt, "status": "ok"}))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle CPU work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["linear", "moe"], default="linear",
                    help="linear: the FP8 linear layer (the headline); moe: the grouped MoE Fprop")
    ap.add_argument("--separate-quant", action="store_true",
                    help="quantise X and dY with separate 1x128 and 128x1 launches")
    ap.add_argument("--profile-gemms", choices=["fp32", "ue8m0"], default=None,
                    help="no timing: quantise the layer once with this scale format, launch its Fprop, "
                         "Dgrad and Wgrad GEMMs once each and exit (a small, fixed launch list for ncu)")
    ap.add_argument("--profile-moe", type=int, default=None, metavar="EXPERTS",
                    help="no timing: one launch of the grouped MoE Fprop GEMM over this many experts (for a "
                         "profiler capture) and exit")
    args = ap.parse_args()
    if args.profile_moe:
        profile_moe(args.profile_moe)
        return
    if args.profile_gemms:
        profile_gemms(args.profile_gemms)
        return
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        line = (run_moe if args.workload == "moe" else run_ours)(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
