"""The multi-GPU split of the path, run through the library on one GPU.

The GEMMs have no exchange step, so a job on several GPUs is a set of
independent problems, one per rank: N slices of a dense problem (whole
128-column scale blocks) or the experts of a grouped problem (balanced by
valid rows, each rank's contiguous layout re-padded to 128 rows).  Here two
ranks are played one after the other on one GPU, through libdg.so, with the
benchmark's own sharding; their outputs, scattered back, must equal the
oracle's unsharded result within the BF16 tolerance, and rows no rank owns
must stay untouched.
"""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import shard, synth

from helpers import bits, check_close, packed, to_device

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu
SENTINEL = 0xDEAD
WORLD = 2


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.set_config(0)
    dg.get_device_error()
    yield


def _run(q):
    t = to_device(q)
    if q.kind == "dense":
        d = dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"])
    elif q.kind == "contiguous":
        d = torch.from_numpy(np.full((q.M, q.N), SENTINEL, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)
        dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"], d)
    else:
        d = torch.from_numpy(np.full((q.G, q.M, q.N), SENTINEL, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)
        dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], t["masked_m"], d)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    return bits(d)


def test_dense_n_split():
    p = synth.dense_problem(384, 1408, 1024, seed=31)   # 11 column blocks: ranks get 5 and 6
    sa, sb = packed(p)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, p.M, p.N, p.K)
    got = np.zeros_like(ref)
    for r in range(WORLD):
        n0, n1 = shard.split_n(p.N, WORLD, r)
        got[:, n0:n1] = _run(bench.shard_problem(p, WORLD, r, "n"))
    check_close(got, ref, "dense, N split over two ranks")


@pytest.mark.parametrize("how", ["n", "experts"])
def test_contiguous_split(how):
    p = synth.contiguous_problem(5, 512, 1024, rows=1500, seed=32)
    sa, sb = packed(p)
    ref = np.full((p.M, p.N), SENTINEL, np.uint16)
    oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, sa, p.b, sb, p.m_indices, ref, p.G, p.N, p.K)
    got = np.full_like(ref, SENTINEL)
    counts = np.bincount(p.m_indices[p.m_indices >= 0], minlength=p.G)
    for r in range(WORLD):
        q = bench.shard_problem(p, WORLD, r, how)
        out = _run(q)
        if how == "n":
            n0, n1 = shard.split_n(p.N, WORLD, r)
            got[:, n0:n1] = out
        else:
            owned = shard.partition_experts(counts, WORLD)[r]
            src, loc = shard.local_contiguous_layout(p.m_indices, owned)
            assert (out[src < 0] == SENTINEL).all(), "local padding rows were written"
            got[src[src >= 0]] = out[src >= 0]
    valid = p.m_indices >= 0
    assert (got[~valid] == SENTINEL).all()
    check_close(got[valid], ref[valid], f"contiguous, split by {how}")


@pytest.mark.parametrize("how", ["n", "experts"])
def test_masked_split(how):
    p = synth.masked_problem(6, 192, 640, 1024, seed=33, masked_m=[0, 191, 64, 3, 129, 192])
    sa, sb = packed(p)
    ref = np.full((p.G, p.M, p.N), SENTINEL, np.uint16)
    oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, p.masked_m, ref, p.G, p.M, p.N, p.K)
    got = np.full_like(ref, SENTINEL)
    for r in range(WORLD):
        out = _run(bench.shard_problem(p, WORLD, r, how))
        if how == "n":
            n0, n1 = shard.split_n(p.N, WORLD, r)
            got[:, :, n0:n1] = out
        else:
            got[shard.partition_experts(p.masked_m, WORLD)[r]] = out
    assert np.array_equal(got == SENTINEL, ref == SENTINEL), "masked rows written, or valid rows missing"
    rows = [(g, m) for g in range(p.G) for m in range(p.masked_m[g])]
    check_close(np.stack([got[g, m] for g, m in rows]), np.stack([ref[g, m] for g, m in rows]),
                f"masked, split by {how}")
