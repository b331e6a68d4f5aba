"""Times the MoE permutation and the weighted combine on their own.

    python -m moe_grouped_gemm_05_b200.moe_timing --op permute [--tokens T --topk k --experts G --k K]
    python -m moe_grouped_gemm_05_b200.moe_timing --op combine [--tokens T --topk k --n N]

Seeded synthetic inputs of the MoE workload (Zipf-skewed top-k routing over
the experts, normal activations quantised to E4M3 with 1x128 scales for the
permutation; BF16 expert outputs and FP32 gate weights for the combine), a few
warm-up calls, then `--iters` calls back to back on the current stream timed
with CUDA events.  Prints the time per call and the device error word.  It is
also the command that the ncu launch lists of these kernels are taken on.
"""
import argparse
import sys

import torch

from . import binding as dg
from . import synth


def _args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--op", choices=["permute", "combine"], required=True)
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--topk", type=int, default=2)
    ap.add_argument("--experts", type=int, default=8, help="experts (permute)")
    ap.add_argument("--k", type=int, default=7168, help="hidden size K of the activations (permute)")
    ap.add_argument("--n", type=int, default=4096, help="columns N of the expert outputs (combine)")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--seed", type=int, default=2002)
    return ap.parse_args(argv)


def main(argv=None) -> int:
    a = _args(argv)
    if not torch.cuda.is_available():
        print("a CUDA device is required", file=sys.stderr)
        return 2
    dev = "cuda"
    gen = torch.Generator(device=dev)
    gen.manual_seed(a.seed + 1)
    T, topk = a.tokens, a.topk
    if a.op == "permute":
        ids, _ = synth.topk_routing(a.seed, T, topk, a.experts)
        ids_d = torch.from_numpy(ids).to(dev)
        x = torch.randn((T, a.k), generator=gen, device=dev).to(torch.bfloat16)
        q, sfa = dg.quantize_fp8_1x128(x)
        out = dg.moe_permute(ids_d, a.experts, q, sfa)

        def call():
            dg.moe_permute(ids_d, a.experts, q, sfa, out=out)
    else:
        rows = T * topk + 1024
        d = torch.randn((rows, a.n), generator=gen, device=dev).to(torch.bfloat16)
        row_of = torch.randperm(rows, generator=gen, device=dev)[: T * topk].reshape(T, topk).to(torch.int32)
        row_of = row_of.contiguous()
        w = torch.rand((T, topk), generator=gen, device=dev)
        out = dg.moe_unpermute_combine(d, row_of, w)

        def call():
            dg.moe_unpermute_combine(d, row_of, w, out=out)
    for _ in range(a.warmup):
        call()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(a.iters):
        call()
    e.record()
    torch.cuda.synchronize()
    err = dg.get_device_error()
    print(f"{a.op}: {s.elapsed_time(e) / a.iters * 1e3:.2f} us per call (T={T}, top-{topk}); device error {err}")
    return 0 if err == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
