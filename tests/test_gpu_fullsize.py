"""Parity at the benchmark workloads' full sizes, in the launch configuration
the benchmark uses (the heuristic's choice, scales packed on the GPU).

The oracle recomputes sampled output rows (first/last rows, tile and expert
boundaries, outlier rows, random rows) in full; properties that hold at any
size (finite outputs, untouched padding / masked rows, bit-exact scale
packing) are checked over the whole output.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close

pytestmark = pytest.mark.gpu

SENTINEL = 0xDEAD


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.set_config(0)
    dg.get_device_error()
    yield
    torch.cuda.empty_cache()


def _pack_on_gpu(sf: np.ndarray):
    """Packs fp32 scales on the GPU and checks the words against the oracle's."""
    sf3 = sf if sf.ndim == 3 else sf[None]
    ref, bad = oracle.pack_sf_ue8m0(sf3)
    assert bad == 0
    got = dg.pack_sf_ue8m0(torch.from_numpy(np.ascontiguousarray(sf3)).cuda())
    assert np.array_equal(got.cpu().numpy(), ref), "GPU scale packing differs from the oracle"
    return got if sf.ndim == 3 else got[0], (ref if sf.ndim == 3 else ref[0])


def _sample_rows(M, rng, extra=()):
    base = {0, 1, 127, 128, 255, 256, M // 2, M - 129, M - 128, M - 2, M - 1, *extra}
    base |= set(rng.integers(0, M, size=12).tolist())
    return np.array(sorted(r for r in base if 0 <= r < M))


def _fp8(x):
    return torch.from_numpy(x).cuda().view(torch.float8_e4m3fn)


@pytest.mark.parametrize("name", ["dense_4096x7168x2048", "dense_64x7168x2048", "dense_8192x8192x8192_outliers"])
def test_dense_full_size(name):
    p = synth.WORKLOADS[name]()
    sfa, sa = _pack_on_gpu(p.sfa)
    sfb, sb = _pack_on_gpu(p.sfb)
    d = dg.fp8_gemm_nt(_fp8(p.a), sfa, _fp8(p.b), sfb)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    got = bits(d)
    assert np.isfinite(oracle.bf16_bits_to_f64(got)).all()
    rng = np.random.default_rng(7)
    extra = ()
    if "outliers" in name:
        # rows scaled by 64 before quantisation (the same draw as the generator's)
        extra = tuple(synth.choose_rows(1004 ^ 0x5A5A, p.M, int(round(0.01 * p.M)))[:6].tolist())
    rows = np.arange(p.M) if p.M <= 64 else _sample_rows(p.M, rng, extra)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, p.M, p.N, p.K, rows=rows)
    check_close(got[rows], ref, name)


def test_contiguous_full_size():
    p = synth.WORKLOADS["contiguous_8x4096x7168_zipf1.1"]()
    sfa, sa = _pack_on_gpu(p.sfa)
    sfb, sb = _pack_on_gpu(p.sfb)
    d = torch.from_numpy(np.full((p.M, p.N), SENTINEL, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)
    dg.m_grouped_fp8_gemm_nt_contiguous(_fp8(p.a), sfa, _fp8(p.b), sfb, torch.from_numpy(p.m_indices).cuda(), d)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    got = bits(d)
    pad = p.m_indices < 0
    assert (got[pad] == SENTINEL).all(), "padding rows were written"
    assert np.isfinite(oracle.bf16_bits_to_f64(got[~pad])).all()
    rng = np.random.default_rng(8)
    rows = []
    for e in range(p.G):
        idx = np.nonzero(p.m_indices == e)[0]
        rows += [idx[0], idx[-1], *rng.choice(idx, size=3, replace=False)]
    rows = np.array(sorted(set(int(r) for r in rows)))
    for e in range(p.G):
        re = rows[p.m_indices[rows] == e]
        ref = oracle.fp8_gemm_nt(p.a, sa, p.b[e], sb[e], p.M, p.N, p.K, rows=re)
        check_close(got[re], ref, f"contiguous expert {e}")


def test_masked_full_size():
    p = synth.WORKLOADS["masked_16x256x7168x2048"]()
    sfa, sa = _pack_on_gpu(p.sfa)
    sfb, sb = _pack_on_gpu(p.sfb)
    d = torch.from_numpy(np.full((p.G, p.M, p.N), SENTINEL, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)
    dg.m_grouped_fp8_gemm_nt_masked(_fp8(p.a), sfa, _fp8(p.b), sfb, torch.from_numpy(p.masked_m).cuda(), d)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    got = bits(d)
    rng = np.random.default_rng(9)
    for g, mg in enumerate(p.masked_m):
        assert (got[g, mg:] == SENTINEL).all(), f"expert {g}: masked rows were written"
        if mg == 0:
            continue
        rows = np.array(sorted({0, mg - 1, *rng.integers(0, mg, size=2).tolist()}))
        ref = oracle.fp8_gemm_nt(p.a[g], sa[g], p.b[g], sb[g], p.M, p.N, p.K, rows=rows)
        check_close(got[g, rows], ref, f"masked expert {g}")
