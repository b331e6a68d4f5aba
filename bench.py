#!/usr/bin/env python
"""Benchmark of the FP8 block-scaled GEMM hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
pack the activation scales (fp32 power-of-two -> UE8M0 int32, the packing
kernel) and run the GEMM (TMA ring -> block-scaled tcgen05 MMA -> epilogue)
on them (--fused-pack: the GEMM reads the fp32 scales and its scale-producer
warp packs them, one launch per step).  Weight scales are packed once, as a
deployment would.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--workloads all|none|a,b]
                    [--impl ours|reference]

Prints ONE JSON line on rank 0.  Its top level is the headline workload,
the largest of the five (the contiguous M-grouped GEMM, 8 experts, 32768
Zipf-routed rows, N=4096, K=7168); with one GPU the same line carries a
``workloads`` object with every workload measured in the same run (kernel
configuration, time, TFLOPS, roofline fraction and the CPU oracle's rate).

With N > 1 (torchrun, one process per GPU) the ranks share one problem
with no collective on the data path; time = max over ranks.  By default
(weak scaling) the problem grows with the ranks: it is the headline problem
widened P-fold along N, each rank owning an N-column block of every
expert's weights and of D (``--shard experts``: P times the experts, each
rank owning the headline's experts and their routed rows), so every rank
runs the headline shape.  ``--scaling strong`` splits the headline problem
itself instead (N in whole 128-column blocks, or the experts).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 block-scaled GEMM TFLOPS (dense/grouped/masked) and % of B200 roofline"
DEFAULT_WORKLOAD = "contiguous_8x4096x7168_zipf1.1"
ALL_WORKLOADS = ("dense_128x512x512", "dense_4096x7168x2048", "dense_64x7168x2048",
                 "contiguous_8x4096x7168_zipf1.1", "masked_16x256x7168x2048", "dense_8192x8192x8192_outliers")
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, help="the headline workload (top level of the line)")
    ap.add_argument("--workloads", default="all",
                    help="workloads measured into the line's 'workloads' object at N=1: all, none or a comma list")
    ap.add_argument("--shard", choices=["n", "experts"], default="n",
                    help="N > 1: split N across ranks (default) or, for grouped workloads, the experts")
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="N > 1: each rank owns a headline-sized share of a P-times larger problem (weak), "
                         "or a 1/P share of the headline problem (strong)")
    ap.add_argument("--min-window-ms", type=float, default=200.0,
                    help="each timing is repeated (K-step graph replays) until this much device time is covered")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the next-row measurements (quantisation, MoE permute/combine, layouts, FP32 + C, 1D1D)")
    ap.add_argument("--next-cpu-seconds", type=float, default=1.5, help="oracle time of each next row's CPU sample")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the headline's oracle sample")
    ap.add_argument("--e2e-steps", type=int, default=0, help="steps of the end-to-end loop (0 = min(steps, 100))")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end loop (profiling runs)")
    ap.add_argument("--eager", action="store_true", help="time host-issued launches instead of a CUDA graph")
    ap.add_argument("--no-library", action="store_true", help="skip the cuBLAS context timing of dense workloads")
    ap.add_argument("--fused-pack", action="store_true",
                    help="let the GEMM read A's fp32 scales and pack them itself instead of a packing launch")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


GEMM_KERNEL_SOURCES = ("fp8_gemm_kernel.cuh", "ptx.cuh")


def kernel_source_hash() -> str:
    """Hash of the GEMM kernel's device code (the host code is covered by the recorded configuration)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_grouped_gemm_05_b200", "csrc")
    for name in GEMM_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel_config: str):
    """Per-launch DRAM bytes of the GEMM kernel from a committed ncu summary,
    only if it was taken on the current kernel code in the same configuration."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(workload)
    if not ent or ent.get("kernel_hash") != kernel_source_hash() or ent.get("kernel_config") != kernel_config:
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, torch_dev: int):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    self._handle = h
                    break
            if self._handle is None:
                self._handle = pynvml.nvmlDeviceGetHandleByIndex(torch_dev)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clock sampling is best effort (NVML may be absent)
            self._handle = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._handle)
                self.samples.append((time.time(), mhz, int(rs)))
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(0.02)

    def start(self):
        if self._handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        busy = [s for s in self.samples if not (s[2] & 0x1)] or self.samples
        bits = 0
        for s in busy:
            bits |= s[2]
        return {"sm_mhz": float(statistics.median(s[1] for s in busy)), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in REASONS.items() if bits & b and b != 0x1], "samples": len(busy)}


# ---------------------------------------------------------------- problems


def algorithmic_bytes(p) -> float:
    """Bytes the GEMM must move at least once: the valid A rows read, B read for
    every expert that has rows, the valid D rows written (BF16), and one UE8M0
    byte per scale of those A rows and B blocks.  Padding and masked-out rows
    cost nothing here, as they do nothing useful."""
    kb = p.K // 128
    nb = (p.N + 127) // 128
    rows = p.valid_rows
    if p.kind == "dense":
        experts = 1
    elif p.kind == "contiguous":
        experts = len(np.unique(p.m_indices[p.m_indices >= 0]))
    else:
        experts = int((p.masked_m > 0).sum())
    return rows * (p.K + kb) + experts * (p.N * p.K + nb * kb) + 2.0 * rows * p.N


def bound_of(p) -> str:
    flops = p.flops
    return "tensor" if flops / algorithmic_bytes(p) > 560.0 else "hbm"


def make_device_sets(p, dg, torch, dev):
    """Device copies of one problem; enough copies that their total exceeds 2x L2."""
    from moe_grouped_gemm_05_b200 import binding

    a = torch.from_numpy(p.a).to(dev).view(torch.float8_e4m3fn)
    b = torch.from_numpy(p.b).to(dev).view(torch.float8_e4m3fn)
    sfa32 = torch.from_numpy(np.ascontiguousarray(p.sfa)).to(dev)
    sfb32 = torch.from_numpy(np.ascontiguousarray(p.sfb)).to(dev)
    if p.kind == "dense":
        d_shape = (p.M, p.N)
    elif p.kind == "contiguous":
        d_shape = (p.M, p.N)
    else:
        d_shape = (p.G, p.M, p.N)
    per_set = a.numel() + b.numel() + 2 * int(np.prod(d_shape))
    nsets = max(1, -(-2 * L2_BYTES // per_set))
    sets = []
    for i in range(nsets):
        s = {"a": a if i == 0 else a.clone(), "b": b if i == 0 else b.clone(),
             "sfa32": sfa32 if i == 0 else sfa32.clone(),
             "d": torch.empty(d_shape, dtype=torch.bfloat16, device=dev)}
        s["sfb"] = binding.pack_sf_ue8m0(sfb32 if i == 0 else sfb32.clone())
        s["sfa"] = binding.pack_sf_ue8m0(s["sfa32"])
        if p.m_indices is not None:
            s["m_indices"] = torch.from_numpy(p.m_indices).to(dev)
        if p.masked_m is not None:
            s["masked_m"] = torch.from_numpy(p.masked_m).to(dev)
        sets.append(s)
    return sets, per_set


def gemm_call(p, dg, s, fp32_sfa=False):
    """The GEMM of a step; with fp32_sfa it reads A's fp32 scales and packs them itself."""
    sfa = s["sfa32"] if fp32_sfa else s["sfa"]
    if p.kind == "dense":
        return dg.fp8_gemm_nt(s["a"], sfa, s["b"], s["sfb"], s["d"])
    if p.kind == "contiguous":
        return dg.m_grouped_fp8_gemm_nt_contiguous(s["a"], sfa, s["b"], s["sfb"], s["m_indices"], s["d"])
    return dg.m_grouped_fp8_gemm_nt_masked(s["a"], sfa, s["b"], s["sfb"], s["masked_m"], s["d"])


def pack_call(dg, lib, s, torch):
    """Packs the step's activation scales into s['sfa'] (the packing kernel, in place)."""
    import ctypes

    sf = s["sfa32"]
    if sf.dim() == 2:
        batch, mn, kb = 1, sf.shape[0], sf.shape[1]
    else:
        batch, mn, kb = sf.shape
    code = lib.dg_pack_sf_ue8m0(ctypes.c_void_p(sf.data_ptr()), ctypes.c_void_p(s["sfa"].data_ptr()), batch, mn,
                                kb, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if code != 0:
        raise RuntimeError(lib.dg_get_last_error().decode())


# ---------------------------------------------------------------- CPU oracle sample


class OracleSample:
    """The CPU oracle on a bounded row sample of a workload (all N, all K).

    One run packs the sample rows' activation scales and computes their
    output rows, i.e. the same two steps as one GPU step, on fewer rows."""

    def __init__(self, p):
        import oracle

        self.oracle, self.p = oracle, p
        if p.kind == "masked":
            g = int(np.argmax(p.masked_m))
            self.a, self.b, self.sfa32, sfb = p.a[g], p.b[g], p.sfa[g], p.sfb[g]
            self.rows_total, self.desc = int(p.masked_m[g]), f"expert {g}"
        elif p.kind == "contiguous":
            self.a, self.b, self.sfa32, sfb = p.a, p.b[0], p.sfa, p.sfb[0]
            self.rows_total, self.desc = int((p.m_indices == 0).sum()), "expert 0"
        else:
            self.a, self.b, self.sfa32, sfb = p.a, p.b, p.sfa, p.sfb
            self.rows_total, self.desc = p.M, "the problem"
        self.sfb = oracle.pack_sf_ue8m0(sfb[None])[0][0]  # weights: packed once
        try:
            from threadpoolctl import threadpool_info

            self.cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:  # noqa: BLE001
            self.cores = os.cpu_count() or 1

    def run(self, rows: int) -> float:
        p, o = self.p, self.oracle
        t0 = time.perf_counter()
        sfa = o.pack_sf_ue8m0(self.sfa32[None, :rows])[0][0]
        o.fp8_gemm_nt(self.a[:rows], sfa, self.b, self.sfb, rows, p.N, p.K)
        return time.perf_counter() - t0

    def calibrate(self, seconds: float) -> int:
        """Rows whose run takes about `seconds` (grown until a run is long enough to extrapolate)."""
        rows = max(1, min(self.rows_total, 16))
        while True:
            t = self.run(rows)
            if rows >= self.rows_total or t >= 0.25 * seconds:
                break
            rows = min(self.rows_total, rows * 4)
        return int(max(1, min(self.rows_total, rows * seconds / max(t, 1e-6))))

    def info(self, rows: int, t: float) -> dict:
        p = self.p
        return {"value": 2.0 * rows * p.N * p.K / t / 1e12, "unit": "TFLOPS", "cores": int(self.cores),
                "kind": "oracle",
                "sample": f"{p.name}: first {rows} valid rows of {self.desc} x all {p.N} columns x K={p.K}, "
                          f"{t:.2f} s per run on host cores"}


# ---------------------------------------------------------------- arms


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from moe_grouped_gemm_05_b200 import synth

    p = synth.WORKLOADS[args.workload]()
    total_steps = args.steps + args.warmup
    per_step = max(0.05, min(2.0, 150.0 / max(total_steps, 1)))
    smp = OracleSample(p)
    rows = smp.calibrate(per_step)
    times = []
    for i in range(total_steps):
        dt = smp.run(rows)
        if i >= args.warmup:
            times.append(dt)
    step_s = statistics.mean(times) if times else smp.run(rows)
    info = smp.info(rows, step_s)
    value = info["value"]
    line = {"metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample_rows": rows, "N": p.N, "K": p.K},
            "impl": "reference", "cpu_baseline": info,
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def global_problem(p, world: int, how: str) -> dict:
    """The whole job's problem under weak scaling: `p` (the headline problem)
    is every rank's share of a problem P times larger along N ("n") or in
    experts and their routed rows ("experts", grouped problems)."""
    g = {"kind": p.kind, "M": p.M, "N": p.N, "K": p.K, "G": p.G, "valid_rows": p.valid_rows}
    if world > 1:
        if how == "experts" and p.kind != "dense":
            g["G"] = p.G * world
            if p.kind == "contiguous":
                g["M"], g["valid_rows"] = p.M * world, p.valid_rows * world
            else:
                g["valid_rows"] = p.valid_rows * world
        else:
            g["N"] = p.N * world
    g["flops"] = p.flops * world
    return g


def shard_problem(p, world: int, rank: int, how: str):
    """This rank's share of problem `p` (strong scaling, no exchange step).

    "n": columns [n0, n1) of every expert in whole 128-column blocks (A and
    the routing are replicated); "experts" (grouped problems): the experts
    ``shard.partition_experts`` gives this rank, re-laid out with
    ``shard.local_contiguous_layout`` (contiguous) or selected (masked)."""
    import dataclasses

    from moe_grouped_gemm_05_b200 import shard

    if world == 1:
        return p
    if how == "experts" and p.kind != "dense":
        if p.kind == "contiguous":
            counts = np.bincount(p.m_indices[p.m_indices >= 0], minlength=p.G)
            owned = shard.partition_experts(counts, world)[rank]
            src, loc = shard.local_contiguous_layout(p.m_indices, owned)
            keep = src >= 0
            a = np.zeros((len(src), p.K), np.uint8)
            a[keep] = p.a[src[keep]]
            sfa = np.ones((len(src), p.sfa.shape[1]), np.float32)
            sfa[keep] = p.sfa[src[keep]]
            return dataclasses.replace(p, a=a, sfa=sfa, b=p.b[owned], sfb=p.sfb[owned], M=len(src), G=len(owned),
                                       m_indices=loc.astype(np.int32), name=f"{p.name}_experts{rank}of{world}")
        owned = shard.partition_experts(p.masked_m, world)[rank]
        return dataclasses.replace(p, a=p.a[owned], sfa=p.sfa[owned], b=p.b[owned], sfb=p.sfb[owned], G=len(owned),
                                   masked_m=p.masked_m[owned], name=f"{p.name}_experts{rank}of{world}")
    n0, n1 = shard.split_n(p.N, world, rank)
    b = np.ascontiguousarray(p.b[..., n0:n1, :])
    sfb = np.ascontiguousarray(p.sfb[..., n0 // 128:(n1 + 127) // 128, :])
    return dataclasses.replace(p, b=b, sfb=sfb, N=n1 - n0, name=f"{p.name}_n{n0}-{n1}")


class Measured(dict):
    pass


def measure(p, dg, lib, torch, args, dev, local, barrier):
    """Times K steps (pack + GEMM) and K GEMM launches of problem `p`.

    Each timing is a CUDA-graph replay of the K launches (or host-issued
    launches with --eager), bracketed by events on the launching stream;
    replays are repeated until --min-window-ms of device time is covered,
    and the median replay is reported.  Step and GEMM-only replays alternate,
    so both medians come from the same stretch of clocks.  Inputs rotate over
    enough device copies that their total exceeds 2x L2.  NVML clocks are sampled during
    the replays."""
    sets, per_set = make_device_sets(p, dg, torch, dev)
    nsets = len(sets)
    fused = args.fused_pack
    K = args.steps

    def step(i):
        s = sets[i % nsets]
        if not fused:
            pack_call(dg, lib, s, torch)
        gemm_call(p, dg, s, fp32_sfa=fused)

    def gemm_only(i):
        gemm_call(p, dg, sets[i % nsets], fp32_sfa=fused)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0, f"{p.name}: device error word set during warm-up"
    kernel_desc = dg.describe_config(p.kind, p.M, p.N, p.K, p.G)

    graphs = {}
    if not args.eager:
        cap = torch.cuda.Stream()
        with torch.cuda.stream(cap):
            cap.wait_stream(torch.cuda.current_stream())
            for name, fn in (("step", step), ("gemm", gemm_only)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    for i in range(K):
                        fn(i)
                graphs[name] = g
        torch.cuda.synchronize()
        for g in graphs.values():  # upload + untimed pass
            g.replay()
        torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def timed(name, fn):
        """Median device time (ms) of one replay of K launches, and the replay count."""
        def once():
            if name in graphs:
                graphs[name].replay()
            else:
                for i in range(K):
                    fn(i)
        ev = []
        total_ms, reps = 0.0, 0
        barrier()
        torch.cuda.synchronize()
        while reps < 3 or (total_ms < args.min_window_ms and reps < 5000):
            batch = max(1, min(64, reps + 1))
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(batch)]
            for a, b in pairs:
                a.record(stream)
                once()
                b.record(stream)
            torch.cuda.synchronize()
            for a, b in pairs:
                ev.append(a.elapsed_time(b))
            total_ms = sum(ev)
            reps = len(ev)
        barrier()
        return statistics.median(ev), reps

    def timed_both():
        """Median device time (ms) of one replay of K steps and of K GEMM launches,
        the two alternating replay by replay so that both see the same clocks
        (under the power cap the SM clock drifts over a window of seconds)."""
        fns = {"step": step, "gemm": gemm_only}
        ev = {n: [] for n in fns}

        def once(name):
            if name in graphs:
                graphs[name].replay()
            else:
                for i in range(K):
                    fns[name](i)
        barrier()
        torch.cuda.synchronize()
        while len(ev["step"]) < 3 or (sum(ev["step"]) + sum(ev["gemm"]) < 2 * args.min_window_ms
                                       and len(ev["step"]) < 5000):
            batch = max(1, min(64, len(ev["step"]) + 1))
            recs = []
            for _ in range(batch):
                for name in fns:
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    once(name)
                    b.record(stream)
                    recs.append((name, a, b))
            torch.cuda.synchronize()
            for name, a, b in recs:
                ev[name].append(a.elapsed_time(b))
        barrier()
        return {n: (statistics.median(v), len(v)) for n, v in ev.items()}

    sampler = ClockSampler(local).start()
    both = timed_both()
    step_ms, step_reps = both["step"]
    gemm_ms, gemm_reps = both["gemm"]
    sampler.stop()
    err = dg.get_device_error()
    library = library_context(p, sets, torch, args, timed, graphs) if p.kind == "dense" else None
    m = Measured(p=p, sets=sets, per_set=per_set, nsets=nsets, kernel_desc=kernel_desc,
                 step_ms=step_ms / K, gemm_ms=gemm_ms / K, replays=step_reps, gemm_replays=gemm_reps,
                 window_ms=step_ms * step_reps, clocks=sampler.summary(), device_error=err, library=library)
    del graphs
    return m


def library_context(p, sets, torch, args, timed, graphs):
    """cuBLAS's FP8 GEMM on the same operands, timed the same way, for context.

    PyTorch's _scaled_mm reaches cuBLAS's 1x128 / 128x128 block-scaled FP8
    GEMM only when built against CUDA 12.9 or later; otherwise the closest
    library GEMM is the per-tensor-scaled FP8 one (one scale per operand: less
    work than the block-scaled recipe, so a generous reference).  Never part
    of the measured path; null with the reason when unavailable."""
    if args.eager or args.no_library:
        return None
    try:
        K = args.steps
        one = torch.ones((), device="cuda")
        ops = [(s["a"], s["b"]) for s in sets]

        def call(i):
            a, b = ops[i % len(ops)]
            torch._scaled_mm(a, b.t(), one, one, out_dtype=torch.bfloat16)

        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            for i in range(3):
                call(i)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                for i in range(K):
                    call(i)
        torch.cuda.synchronize()
        graphs["library"] = g
        ms, reps = timed("library", None)
        return {"library": "cuBLAS FP8 GEMM through torch._scaled_mm, per-tensor scales (the block-scaled "
                           "recipe needs CUDA 12.9 in PyTorch's build)", "kernel_ms_avg": ms / K,
                "tflops": p.flops / (ms / K * 1e-3) / 1e12, "replays": reps}
    except Exception as e:  # noqa: BLE001 - context only
        return {"unavailable": f"{type(e).__name__}: {str(e)[:160]}"}


def roofline_of(p, gemm_ms, clocks, window_ms, workload_key, kernel_desc):
    peaks, peak_src = load_peaks()
    bound = bound_of(p)
    # The sustained peak was measured under the power cap: use it when the timed
    # windows were long or the clock sampler saw the cap; the burst peak otherwise.
    power_capped = "sw_power_cap" in clocks.get("reasons", [])
    long_region = window_ms > 500.0 or power_capped
    if bound == "tensor":
        bf16 = peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops")
        peak = 2.0 * bf16  # FP8 dense = 2 x BF16 dense (nominal ratio)
        achieved = p.flops / (gemm_ms * 1e-3) / 1e12
        unit = "TFLOP/s"
        note = (f"{'sustained' if long_region else 'burst'} bf16 x2 ({peak_src} peaks)"
                + ("; power cap active during the timed region" if power_capped else ""))
    else:
        peak = peaks.get("hbm_gbs")
        achieved = algorithmic_bytes(p) / (gemm_ms * 1e-3) / 1e9
        unit = "GB/s"
        note = f"copy bandwidth ({peak_src} peaks)"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak if peak else None, "traffic": recorded_traffic(workload_key, kernel_desc),
            "traffic_note": ("DRAM read + write bytes of one launch from a committed ncu capture of this kernel "
                             "code and configuration; D rows still in L2 when the kernel ends are not counted"),
            "peak_source": note, "kernel": "fp8_gemm_kernel", "kernel_ms_avg": gemm_ms,
            "algorithmic": (f"{p.flops:.4g} FLOP" if bound == "tensor" else f"{algorithmic_bytes(p):.4g} B")
            + " per launch"}


# ---------------------------------------------------------------- the "next" rows

# The MoE step around the contiguous GEMM: 16384 tokens routed top-2 over 8
# experts (Zipf(1.1) weights), hidden K = 7168, expert output N = 4096.
NEXT_T, NEXT_TOPK, NEXT_G, NEXT_K, NEXT_N = 16384, 2, 8, 7168, 4096


def _graph_time(fn, torch, args, local):
    """Median device time (ms) of one launch of fn(i): K launches captured in a
    CUDA graph, replayed until --min-window-ms of device time is covered, with
    the clocks sampled meanwhile.  Returns (ms, replays, window_ms, clocks)."""
    K = args.steps
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for i in range(K):
                fn(i)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local).start()
    ev = []
    while len(ev) < 3 or (sum(ev) < args.min_window_ms and len(ev) < 5000):
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(max(1, min(64, len(ev) + 1)))]
        for a, b in pairs:
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        ev += [a.elapsed_time(b) for a, b in pairs]
    sampler.stop()
    del g
    return statistics.median(ev) / K, len(ev), sum(ev), sampler.summary()


def _cores():
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def _timed_cpu(fn, seconds: float, unit_fn, sample_fn):
    """The oracle on a growing sample until one run takes about `seconds`; returns its rate."""
    n = 1
    while True:
        t0 = time.perf_counter()
        fn(n)
        t = time.perf_counter() - t0
        if t >= 0.25 * seconds or n >= sample_fn(None):
            break
        n = min(sample_fn(None), n * 4)
    n = int(max(1, min(sample_fn(None), n * seconds / max(t, 1e-6))))
    t0 = time.perf_counter()
    fn(n)
    t = time.perf_counter() - t0
    value, unit = unit_fn(n, t)
    return {"value": value, "unit": unit, "cores": int(_cores()), "kind": "oracle", "sample": sample_fn(n) +
            f", {t:.2f} s per run on host cores"}


def _next_row(what, timing, *, flops=None, nbytes=None, cpu=None):
    """One next-row entry: time, roofline (tensor-bound when the FLOP per byte
    exceed the ridge, else HBM-bound) and the oracle's rate."""
    ms, reps, window, clocks = timing
    peaks, src = load_peaks()
    capped = "sw_power_cap" in clocks.get("reasons", [])
    long_region = window > 500.0 or capped
    if flops is not None and (nbytes is None or flops / nbytes > 560.0):
        peak = 2.0 * peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops")
        roof = {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                "algorithmic": f"{flops:.4g} FLOP per launch",
                "peak_source": f"{'sustained' if long_region else 'burst'} bf16 x2 ({src} peaks)"}
    else:
        peak = peaks.get("hbm_gbs")
        roof = {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                "algorithmic": f"{nbytes:.4g} B per launch", "peak_source": f"copy bandwidth ({src} peaks)"}
    roof["frac"] = roof["achieved"] / peak if peak else None
    return {"what": what, "ms_per_launch": ms, "replays": reps, "window_ms": window, "roofline": roof,
            "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")}, "cpu_baseline": cpu}


def measure_next_rows(dg, torch, args, dev, local) -> dict:
    """The rows beyond the GEMM of the headline path, each timed like the
    workloads (CUDA-graph replays, median per launch), against its roofline,
    with the oracle's rate on a bounded sample (--next-cpu-seconds each):
    activation quantisation, the MoE permutation and combine around the
    contiguous GEMM, the NN / TN / TT operand layouts, FP32 output plus C, and
    the 1D1D recipe (both on the dense 4096 x 7168 x 2048 problem)."""
    from oracle import fp8_gemm as oracle
    from moe_grouped_gemm_05_b200 import synth

    secs = 0 if args.no_cpu_baseline else args.next_cpu_seconds
    rows = {}
    gen = torch.Generator(device=dev)
    f8 = torch.float8_e4m3fn

    # activation quantisation: the contiguous workload's 32768 x 7168 BF16 activations
    M, K = 32768, NEXT_K
    gen.manual_seed(2001)
    x = torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16)
    q = torch.empty((M, K), dtype=f8, device=dev)
    sf = torch.empty(dg.packed_sf_words(M, K // 128), dtype=torch.int32, device=dev)
    kp, mn4 = dg.packed_sf_words(M, K // 128)
    t = _graph_time(lambda i: dg.quantize_fp8_1x128(x, q=q, sf=sf), torch, args, local)
    cpu = None
    if secs:
        xs = x[:4096].float().cpu().numpy()
        cpu = _timed_cpu(lambda n: oracle.quantize_fp8_1x128(xs[:n]), secs,
                         lambda n, s: (n * K * 3 / s / 1e9, "GB/s"),
                         lambda n: 4096 if n is None else f"first {n} of the {M} rows x K={K}")
    rows["quantize_fp8_1x128"] = _next_row(f"BF16 [{M}, {K}] -> E4M3 + packed UE8M0 (1x128)", t,
                                           nbytes=M * K * 2 + M * K + 4 * kp * mn4, cpu=cpu)
    del x, q, sf

    # MoE permutation (routing + gather into the contiguous layout) and the weighted combine
    T, topk, G, N = NEXT_T, NEXT_TOPK, NEXT_G, NEXT_N
    ids, gates = synth.topk_routing(2002, T, topk, G)
    ids_d, gates_d = torch.from_numpy(ids).to(dev), torch.from_numpy(gates).to(dev)
    gen.manual_seed(2003)
    qt, sft = dg.quantize_fp8_1x128(torch.randn((T, K), generator=gen, device=dev).to(torch.bfloat16))
    per = dg.moe_permute(ids_d, G, qt, sft)
    cap = per["a"].shape[0]
    routed = T * topk
    kp_t = (K // 128 + 3) // 4
    t = _graph_time(lambda i: dg.moe_permute(ids_d, G, qt, sft, out=per), torch, args, local)
    cpu = None
    if secs:
        qh = qt.view(torch.uint8).cpu().numpy()

        def permute_cpu(n):
            m_idx, row_of, src_of, total, bad = oracle.moe_permute(ids[:n], G)
            return qh[src_of[src_of >= 0]]

        cpu = _timed_cpu(permute_cpu, secs, lambda n, s: (n * topk * K * 2 / s / 1e9, "GB/s"),
                         lambda n: T if n is None else f"first {n} of the {T} tokens (top-{topk} of {G})")
    rows["moe_permute"] = _next_row(
        f"{T} tokens top-{topk} over {G} experts -> contiguous layout ({cap} rows), K={K}", t,
        nbytes=T * K + 4 * T * kp_t + 4 * routed + routed * K + 4 * routed * kp_t + 8 * cap + 4 * routed, cpu=cpu)
    gen.manual_seed(2004)
    dperm = torch.randn((cap, N), generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    t = _graph_time(lambda i: dg.moe_unpermute_combine(dperm, per["row_of"], gates_d, out=out), torch, args, local)
    cpu = None
    if secs:
        row_of = per["row_of"].cpu().numpy()
        d_bits = dperm[:, :].view(torch.int16).cpu().numpy().view(np.uint16)

        def combine_cpu(n):
            r = row_of[:n].reshape(-1)
            return oracle.moe_unpermute_combine(d_bits[r], np.arange(len(r), dtype=np.int32).reshape(n, topk),
                                                gates[:n])

        cpu = _timed_cpu(combine_cpu, secs, lambda n, s: ((n * topk * N * 2 + n * N * 2) / s / 1e9, "GB/s"),
                         lambda n: T if n is None else f"first {n} of the {T} tokens x N={N}")
    rows["moe_unpermute_combine"] = _next_row(f"{T} tokens x top-{topk} BF16 rows of N={N} -> weighted sum", t,
                                              nbytes=routed * N * 2 + 8 * routed + T * N * 2, cpu=cpu)
    del qt, sft, per, dperm, out

    # the dense 4096 x 7168 x 2048 problem in the other operand layouts, FP32 output + C, and 1D1D
    p = synth.WORKLOADS["dense_4096x7168x2048"]()
    M, N, K = p.M, p.N, p.K
    flops = p.flops
    sfa = dg.pack_sf_ue8m0(torch.from_numpy(np.ascontiguousarray(p.sfa)).to(dev))
    sfb = dg.pack_sf_ue8m0(torch.from_numpy(np.ascontiguousarray(p.sfb)).to(dev))
    nsets = 4  # 4 x (A + B + D) = 330 MB > 2x L2
    to = lambda arr: torch.from_numpy(np.ascontiguousarray(arr)).to(dev).view(f8)  # noqa: E731
    gemm_cpu = None
    if secs:
        smp = OracleSample(p)
        r = smp.calibrate(secs)
        gemm_cpu = smp.info(r, smp.run(r))
    for layout in ("nn", "tn", "tt"):
        a_s = to(p.a.T) if layout[0] == "t" else to(p.a)
        b_s = to(p.b.T) if layout[1] == "n" else to(p.b)
        sets = [(a_s if i == 0 else a_s.clone(), b_s if i == 0 else b_s.clone(),
                 torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for i in range(nsets)]
        t = _graph_time(lambda i: dg.fp8_gemm(layout, sets[i % nsets][0], sfa, sets[i % nsets][1], sfb,
                                              sets[i % nsets][2]), torch, args, local)
        rows[f"fp8_gemm_{layout}"] = _next_row(
            f"dense {M}x{N}x{K}, A stored {'[K][M]' if layout[0] == 't' else '[M][K]'}, "
            f"B stored {'[K][N]' if layout[1] == 'n' else '[N][K]'}", t, flops=flops,
            nbytes=M * K + N * K + 2 * M * N, cpu=gemm_cpu)
        del sets, a_s, b_s
    a, b = to(p.a), to(p.b)
    gen.manual_seed(2005)
    c = torch.randn((M, N), generator=gen, device=dev)
    dsets = [torch.empty((M, N), dtype=torch.float32, device=dev) for _ in range(2)]
    t = _graph_time(lambda i: dg.fp8_gemm_nt_ex(a, sfa, b, sfb, c=c, d=dsets[i % 2], out_dtype=torch.float32),
                    torch, args, local)
    cpu = None
    if secs:
        sa_w, sb_w = oracle.pack_sf_ue8m0(p.sfa[None])[0][0], oracle.pack_sf_ue8m0(p.sfb[None])[0][0]
        ch = c[:1024].cpu().numpy()
        cpu = _timed_cpu(lambda n: oracle.fp8_gemm_nt_general_f64(p.a, sa_w, p.b, sb_w, M, N, K, c=ch,
                                                                  rows=np.arange(n)), secs,
                         lambda n, s: (2.0 * n * N * K / s / 1e12, "TFLOPS"),
                         lambda n: 1024 if n is None else f"first {n} rows x all {N} columns x K={K}")
    rows["fp8_gemm_nt_ex_fp32_plus_c"] = _next_row(f"dense {M}x{N}x{K}, FP32 D = A.B^T + C (FP32 C)", t, flops=flops,
                                                   nbytes=M * K + N * K + 8 * M * N, cpu=cpu)
    del c, dsets
    # 1D1D: one scale per row of B (each 128x128 block's scale repeated over its rows)
    sfb_rows = np.ascontiguousarray(np.repeat(p.sfb, 128, axis=0)[:N])
    sfb1 = dg.pack_sf_ue8m0(torch.from_numpy(sfb_rows).to(dev))
    dsets = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(nsets)]
    asets = [a if i == 0 else a.clone() for i in range(nsets)]
    t = _graph_time(lambda i: dg.fp8_gemm_nt_ex(asets[i % nsets], sfa, b, sfb1, d=dsets[i % nsets], recipe_b=1),
                    torch, args, local)
    cpu = None
    if secs:
        sa_w = oracle.pack_sf_ue8m0(p.sfa[None])[0][0]
        sb1_w = oracle.pack_sf_ue8m0(sfb_rows[None])[0][0]
        cpu = _timed_cpu(lambda n: oracle.fp8_gemm_nt_general_f64(p.a, sa_w, p.b, sb1_w, M, N, K, sfb_gran_n=1,
                                                                  rows=np.arange(n)), secs,
                         lambda n, s: (2.0 * n * N * K / s / 1e12, "TFLOPS"),
                         lambda n: 1024 if n is None else f"first {n} rows x all {N} columns x K={K}")
    rows["fp8_gemm_nt_ex_1d1d"] = _next_row(f"dense {M}x{N}x{K}, B with one scale per row and 128-K block", t,
                                            flops=flops, nbytes=M * K + N * K + 2 * M * N, cpu=cpu)
    del asets, dsets, a, b
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0, "device error word set during the next-row measurements"
    torch.cuda.empty_cache()
    return rows


def e2e_loop(p, m, dg, lib, torch, args, barrier):
    """End to end through the public API: every step copies its inputs from
    pinned host memory, packs + multiplies, and copies D back to pinned host
    memory.  When a step moves at least 8 MB, consecutive steps overlap on
    three streams over two device buffer sets (H2D of step i+1 and D2H of
    step i-1 run beside step i's GEMM), as a serving loop would; smaller
    steps, bound by copy-launch latency, run on one stream.  The time runs
    from the first copy in to the last copy out."""
    sets, fused = m["sets"], args.fused_pack
    e2e_steps = args.e2e_steps or min(args.steps, 100)
    if len(sets) > 1:
        bufs = [sets[0], sets[1]]
    else:  # one set is already > 2x L2: a second one for A, its scales and D (B shared)
        s1 = dict(sets[0])
        s1["a"], s1["sfa32"] = sets[0]["a"].clone(), sets[0]["sfa32"].clone()
        s1["sfa"], s1["d"] = sets[0]["sfa"].clone(), torch.empty_like(sets[0]["d"])
        bufs = [sets[0], s1]
    a_host = torch.from_numpy(p.a).pin_memory()
    sfa_host = torch.from_numpy(np.ascontiguousarray(p.sfa)).pin_memory()
    d_host = torch.empty(bufs[0]["d"].shape, dtype=torch.bfloat16).pin_memory()
    h2d = a_host.numel() + sfa_host.numel() * 4
    d2h = d_host.numel() * 2
    overlap = h2d + d2h >= (8 << 20)
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step_serial(i):  # small steps: one stream, no events (host enqueue cost matters)
        sb = bufs[0]
        sb["a"].view(torch.uint8).copy_(a_host, non_blocking=True)
        sb["sfa32"].copy_(sfa_host, non_blocking=True)
        if not fused:
            pack_call(dg, lib, sb, torch)
        gemm_call(p, dg, sb, fp32_sfa=fused)
        d_host.copy_(sb["d"], non_blocking=True)

    def e2e_step_overlap(i):
        b = i % 2
        sb = bufs[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])  # step i-2 has finished reading this set's inputs
            sb["a"].view(torch.uint8).copy_(a_host, non_blocking=True)
            sb["sfa32"].copy_(sfa_host, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_out[b])  # step i-2's D has left this set
            if not fused:
                pack_call(dg, lib, sb, torch)
            gemm_call(p, dg, sb, fp32_sfa=fused)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            d_host.copy_(sb["d"], non_blocking=True)
            ev_out[b].record(s_out)

    e2e_step = e2e_step_overlap if overlap else e2e_step_serial
    first = s_in if overlap else torch.cuda.current_stream()
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(first)
    for i in range(e2e_steps):
        e2e_step(i)
    if overlap:
        s_in.wait_stream(s_out)
    e1.record(first)
    torch.cuda.synchronize()
    barrier()
    return {"ms": e0.elapsed_time(e1), "steps": e2e_steps, "h2d": h2d, "d2h": d2h, "overlap": overlap}


def cpu_baseline_of(p, seconds):
    smp = OracleSample(p)
    rows = smp.calibrate(seconds)
    return smp.info(rows, smp.run(rows))


def run_ours(args):
    import torch
    import torch.distributed as dist

    from moe_grouped_gemm_05_b200 import binding as dg
    from moe_grouped_gemm_05_b200 import shard, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    lib = dg.load()
    full = synth.WORKLOADS[args.workload]()
    weak = args.scaling == "weak"
    # weak: every rank runs the headline shape as its share; strong: a 1/P share of it
    p = full if weak else shard_problem(full, world, rank, args.shard)
    job = global_problem(full, world, args.shard) if weak else global_problem(full, 1, args.shard)
    m = measure(p, dg, lib, torch, args, dev, local, barrier)
    e2e = None if args.no_e2e else e2e_loop(p, m, dg, lib, torch, args, barrier)
    m["sets"] = None
    torch.cuda.empty_cache()

    # max over ranks of every time; the work is the whole job's problem
    step_ms = shard.max_over_ranks(m["step_ms"])
    gemm_ms = shard.max_over_ranks(m["gemm_ms"])
    e2e_ms = shard.max_over_ranks(e2e["ms"]) if e2e else None
    flops = job["flops"]
    value = flops / (step_ms * 1e-3) / 1e12
    # roofline of this rank's kernel on this rank's share (rank 0 reports it)
    roof = roofline_of(p, m["gemm_ms"], m["clocks"], m["window_ms"],
                       args.workload if (world == 1 or weak) else p.name, m["kernel_desc"])
    clocks = m["clocks"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak" if (weak or world == 1) else "strong", "vs_baseline": None, "dtype": "fp8_e4m3",
        "data": "synthetic",
        "config": {"workload": args.workload, "kind": full.kind, "M": full.M, "N": full.N, "K": full.K, "G": full.G,
                   "valid_rows": full.valid_rows, "kernel_config": m["kernel_desc"],
                   "parallelism": (f"{world} ranks, " + ("N split" if args.shard == "n" or full.kind == "dense"
                                                         else "experts split")
                                   + (f", each rank owning a {full.name} share of a {world}x larger problem"
                                      if weak else " of the headline problem in 128-column blocks / expert sets")
                                   if world > 1 else "one GPU"),
                   "step": ("GEMM reading A's fp32 scales, packed to UE8M0 in its scale-producer warp"
                            if args.fused_pack else "pack activation scales (fp32 -> UE8M0 int32) + GEMM"),
                   "timing": (("eager launches" if args.eager else "CUDA-graph replay of the K steps")
                              + f"; median of {m['replays']} replays ({m['window_ms']:.0f} ms of device time),"
                              + " alternating with the GEMM-only replays that give the roofline's kernel time"),
                   "l2": (f"inputs rotate over {m['nsets']} device copies "
                          f"({m['nsets'] * m['per_set'] / 1e6:.0f} MB > 2x L2)")},
        "roofline": roof,
        # this library's launches in one replay of the K steps (the replay whose time is ms_per_step x steps)
        "gpu_launches": (1 if args.fused_pack else 2) * args.steps,
        "gpu_launches_note": (f"per replay of the {args.steps} steps; the reported time is the median of "
                              f"{m['replays']} replays"),
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "device_error": m["device_error"],
    }
    if world > 1:
        # the whole job's problem; with weak scaling every rank's share holds the headline problem's values
        line["config"]["job_problem"] = {k: v for k, v in job.items() if k != "flops"}
        line["config"]["job_flop"] = job["flops"]
    if e2e:
        line["e2e"] = {"value": flops * e2e["steps"] / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["steps"],
                       "overlap": ("H2D / compute / D2H of consecutive steps on three streams" if e2e["overlap"]
                                   else "none: one stream (less than 8 MB of copies per step)")}

    # every workload in the same run (one GPU): kernel configuration, time, rate, roofline, CPU oracle
    names = []
    if world == 1 and args.workloads != "none":
        names = list(ALL_WORKLOADS) if args.workloads == "all" else args.workloads.split(",")
    if names:
        line["workloads"] = {}
    for name in names:
        if name == args.workload:
            q, mq = full, m
        else:
            q = synth.WORKLOADS[name]()
            mq = measure(q, dg, lib, torch, args, dev, local, barrier)
            mq["sets"] = None
            torch.cuda.empty_cache()
        entry = {"kind": q.kind, "M": q.M, "N": q.N, "K": q.K, "G": q.G, "valid_rows": q.valid_rows,
                 "kernel_config": mq["kernel_desc"], "ms_per_step": mq["step_ms"], "kernel_ms_avg": mq["gemm_ms"],
                 "value": q.flops / (mq["step_ms"] * 1e-3) / 1e12, "unit": "TFLOPS",
                 "kernel_tflops": q.flops / (mq["gemm_ms"] * 1e-3) / 1e12,
                 "roofline": roofline_of(q, mq["gemm_ms"], mq["clocks"], mq["window_ms"], name, mq["kernel_desc"]),
                 "replays": mq["replays"], "window_ms": mq["window_ms"],
                 "library_context": mq["library"],
                 "clocks": {k: mq["clocks"][k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
                 "device_error": mq["device_error"]}
        if not args.no_cpu_baseline:
            secs = args.cpu_seconds if name == args.workload else max(1.0, args.cpu_seconds / 2)
            entry["cpu_baseline"] = cpu_baseline_of(q, secs)
            if name == args.workload:
                line["cpu_baseline"] = entry["cpu_baseline"]
        line["workloads"][name] = entry
    if rank == 0 and world == 1 and not args.no_cpu_baseline and "cpu_baseline" not in line:
        line["cpu_baseline"] = cpu_baseline_of(full, args.cpu_seconds)
    # the rows beyond the headline's GEMM (one GPU, full runs only)
    if world == 1 and args.workloads != "none" and not args.no_next_rows and not args.eager:
        line["next_rows"] = measure_next_rows(dg, torch, args, dev, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
