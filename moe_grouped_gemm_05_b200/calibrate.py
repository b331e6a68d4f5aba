"""Times every built tile configuration on a set of workloads, on the GPU.

This produces the measurements that the configuration heuristic's cost model
(``csrc/dg_api.cu``: ``kCost``, ``kCostContig``) was fitted to, so that they
can be re-taken on another GPU or after a kernel change:

    python -m moe_grouped_gemm_05_b200.calibrate [--workloads a,b,...] [--rounds R] [--launches L]

For each workload every configuration is forced in turn (``dg_set_config``)
and captured as a CUDA graph of L back-to-back GEMM launches on rotating
input copies (more than 2x L2 in total).  The graphs are replayed
round-robin, R rounds, so that every configuration sees the same power and
thermal states; the median over rounds is reported per launch, with the
heuristic's own pick alongside.  With both dense calibration shapes present
(K = 2048 and K = 8192) it also fits, per configuration, the cost model's
time per 128-wide K block of a tile and the time per tile on top of it.

Inputs come from the seeded synthetic workloads of ``synth``; nothing here
checks results (the parity tests do that).
"""
from __future__ import annotations

import argparse
import json
import math
import statistics

import numpy as np

from . import binding as dg
from . import synth

L2_BYTES = 126 * 1024 * 1024

# Built (block_n, ctas, pipes) triples per layout, as listed with dg_set_config in include/dg.h.
CONFIGS = {
    "dense": [(128, 1, 1), (224, 1, 1), (256, 1, 1), (128, 2, 1), (224, 2, 1), (256, 2, 1), (224, 2, 2), (128, 2, 2),
              (64, 1, 1), (64, 1, 2), (128, 1, 2)],
    "masked": [(128, 1, 1), (224, 1, 1), (256, 1, 1), (128, 2, 1), (224, 2, 1), (256, 2, 1), (224, 2, 2), (128, 2, 2),
               (64, 1, 1), (64, 1, 2), (128, 1, 2)],
    "contiguous": [(128, 1, 1), (224, 1, 1), (256, 1, 1), (224, 2, 2)],
}
DEFAULT_WORKLOADS = ("dense_4096x7168x2048", "dense_8192x8192x8192_outliers", "contiguous_8x4096x7168_zipf1.1",
                     "masked_16x256x7168x2048", "dense_64x7168x2048")


def _device_sets(p, torch):
    """Device copies of problem p (packed scales), enough that their total exceeds 2x L2."""
    a = torch.from_numpy(p.a).cuda().view(torch.float8_e4m3fn)
    b = torch.from_numpy(p.b).cuda().view(torch.float8_e4m3fn)
    sfa = dg.pack_sf_ue8m0(torch.from_numpy(np.ascontiguousarray(p.sfa)).cuda())
    sfb = dg.pack_sf_ue8m0(torch.from_numpy(np.ascontiguousarray(p.sfb)).cuda())
    d_shape = (p.G, p.M, p.N) if p.kind == "masked" else (p.M, p.N)
    per_set = a.numel() + b.numel() + 2 * math.prod(d_shape)
    sets = []
    for i in range(max(1, -(-2 * L2_BYTES // per_set))):
        s = {"a": a if i == 0 else a.clone(), "b": b if i == 0 else b.clone(), "sfa": sfa, "sfb": sfb,
             "d": torch.empty(d_shape, dtype=torch.bfloat16, device="cuda")}
        if p.m_indices is not None:
            s["m_indices"] = torch.from_numpy(p.m_indices).cuda()
        if p.masked_m is not None:
            s["masked_m"] = torch.from_numpy(p.masked_m).cuda()
        sets.append(s)
    return sets


def _call(p, s):
    if p.kind == "dense":
        dg.fp8_gemm_nt(s["a"], s["sfa"], s["b"], s["sfb"], s["d"])
    elif p.kind == "contiguous":
        dg.m_grouped_fp8_gemm_nt_contiguous(s["a"], s["sfa"], s["b"], s["sfb"], s["m_indices"], s["d"])
    else:
        dg.m_grouped_fp8_gemm_nt_masked(s["a"], s["sfa"], s["b"], s["sfb"], s["masked_m"], s["d"])


def time_configs(name: str, rounds: int, launches: int) -> dict:
    """Median per-launch time (ms) of every built configuration on one workload, plus the heuristic's."""
    import torch

    p = synth.WORKLOADS[name]()
    sets = _device_sets(p, torch)
    graphs = {}
    for cfg in CONFIGS[p.kind] + [(0, 0, 0)]:
        dg.set_config(*cfg)
        try:
            _call(p, sets[0])
            torch.cuda.synchronize()
            label = "heuristic: " + dg.describe_config(p.kind, p.M, p.N, p.K, p.G) if cfg == (0, 0, 0) else str(cfg)
            cap = torch.cuda.Stream()
            with torch.cuda.stream(cap):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    for i in range(launches):
                        _call(p, sets[i % len(sets)])
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            graphs[label] = g
        finally:
            dg.set_config(0)
    times = {k: [] for k in graphs}
    for _ in range(rounds):
        for label, g in graphs.items():
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            times[label].append(a.elapsed_time(b) / launches)
    assert dg.get_device_error() == 0
    out = {"kind": p.kind, "M": p.M, "N": p.N, "K": p.K, "G": p.G, "flops": p.flops, "ms": {}}
    for label, ts in times.items():
        out["ms"][label] = statistics.median(ts)
    del graphs, sets
    torch.cuda.empty_cache()
    return out


def fit_dense(res: dict, sms: int = 148) -> dict:
    """Per configuration: ns per 128-wide K block of a tile and ns per tile, from the two dense shapes.

    A launch is modelled as (tiles / units) x (K/128 x kb + tile), units = SMs / CTAs per tile;
    split-K tiles run half of the K blocks on each pipeline."""
    a, b = res.get("dense_4096x7168x2048"), res.get("dense_8192x8192x8192_outliers")
    if not a or not b:
        return {}
    fit = {}
    for cfg in CONFIGS["dense"]:
        bn, ctas, pipes = cfg
        split = cfg in ((64, 1, 2), (128, 1, 2))
        per = []
        for r in (a, b):
            tiles = math.ceil(r["M"] / (128 * ctas)) * math.ceil(r["N"] / bn)
            waves = max(1.0, tiles / (sms // ctas))
            kb = r["K"] / 128 / (2 if split else 1)
            per.append((kb, r["ms"][str(cfg)] * 1e6 / waves))
        (k1, t1), (k2, t2) = per
        kb_ns = (t2 - t1) / (k2 - k1)
        fit[str(cfg)] = {"kb_ns": round(kb_ns), "tile_ns": round(t1 - k1 * kb_ns)}
    return fit


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", default=",".join(DEFAULT_WORKLOADS))
    ap.add_argument("--rounds", type=int, default=8)
    ap.add_argument("--launches", type=int, default=10)
    ap.add_argument("--json", default="", help="also write the results to this file")
    args = ap.parse_args()
    res = {}
    for name in args.workloads.split(","):
        res[name] = time_configs(name, args.rounds, args.launches)
        r = res[name]
        print(f"\n{name}  ({r['kind']}, M={r['M']} N={r['N']} K={r['K']} G={r['G']})")
        best = min(v for k, v in r["ms"].items() if not k.startswith("heuristic"))
        for label, ms in sorted(r["ms"].items(), key=lambda kv: kv[1]):
            print(f"  {label:44s} {ms * 1e3:9.2f} us  {r['flops'] / (ms * 1e-3) / 1e12:7.0f} TFLOP/s"
                  f"  {ms / best:5.3f}x best", flush=True)
    fit = fit_dense(res)
    if fit:
        print("\nfit (dense): config -> ns per K block of a tile, ns per tile")
        for k, v in fit.items():
            print(f"  {k:14s} kb {v['kb_ns']:5d}  tile {v['tile_ns']:6d}")
    if args.json:
        with open(args.json, "w") as f:
            json.dump({"results": res, "fit": fit}, f, indent=1)


if __name__ == "__main__":
    main()
