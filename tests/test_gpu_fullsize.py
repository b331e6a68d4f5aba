"""Parity at the benchmark workloads' full sizes, in the launch configuration
the benchmark uses (the heuristic's choice, scales packed on the GPU).

Every valid output row of all five workloads is recomputed by the oracle
(on a thread pool, a chunk of rows per call) and compared element by element
within the BF16 tolerance; padding rows of the contiguous layout and masked
rows keep their sentinel bit pattern, and the scale packing is bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close, oracle_rows

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


def _fp8(x):
    return torch.from_numpy(x).cuda().view(torch.float8_e4m3fn)


def _sentinel(shape):
    return torch.from_numpy(np.full(shape, SENTINEL, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("name", ["dense_4096x7168x2048", "dense_64x7168x2048", "dense_8192x8192x8192_outliers"])
def test_dense_full_size(name):
    p = synth.WORKLOADS[name]()
    sfa, sa = _pack_on_gpu(p.sfa)
    sfb, sb = _pack_on_gpu(p.sfb)
    d = dg.fp8_gemm_nt(_fp8(p.a), sfa, _fp8(p.b), sfb)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    got = bits(d)
    ref = oracle_rows(p.a, sa, p.b, sb, p.M, p.N, p.K, np.arange(p.M))
    check_close(got, ref, name)
    if "outliers" in name:
        # the rows scaled by 64 before quantisation (the generator's own draw) are among them
        out = synth.choose_rows(1004 ^ 0x5A5A, p.M, int(round(0.01 * p.M)))
        assert len(out) == 82
        check_close(got[out], ref[out], f"{name}: outlier rows")


def test_contiguous_full_size():
    """The heuristic's configuration and the 2-CTA tiles whose block pairs the
    kernel forms within each expert's run, both against one oracle result."""
    p = synth.WORKLOADS["contiguous_8x4096x7168_zipf1.1"]()
    sfa, sa = _pack_on_gpu(p.sfa)
    sfb, sb = _pack_on_gpu(p.sfb)
    pad = p.m_indices < 0
    ref = np.full((p.M, p.N), SENTINEL, np.uint16)
    for e in range(p.G):
        rows = np.nonzero(p.m_indices == e)[0]
        assert len(rows) > 0
        ref[rows] = oracle_rows(p.a, sa, p.b[e], sb[e], p.M, p.N, p.K, rows)
    a, b, mi = _fp8(p.a), _fp8(p.b), torch.from_numpy(p.m_indices).cuda()
    for cfg in ((0, 0, 0), (224, 2, 2)):
        dg.set_config(*cfg)
        d = _sentinel((p.M, p.N))
        dg.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, mi, d)
        torch.cuda.synchronize()
        dg.set_config(0)
        assert dg.get_device_error() == 0
        got = bits(d)
        assert (got[pad] == SENTINEL).all(), f"padding rows were written, cfg={cfg}"
        for e in range(p.G):
            rows = np.nonzero(p.m_indices == e)[0]
            check_close(got[rows], ref[rows], f"contiguous expert {e}, cfg={cfg}")
        # the whole call's normalised difference, over every valid row
        check_close(got[~pad], ref[~pad], f"contiguous, all valid rows, cfg={cfg}")


def test_masked_full_size():
    p = synth.WORKLOADS["masked_16x256x7168x2048"]()
    sfa, sa = _pack_on_gpu(p.sfa)
    sfb, sb = _pack_on_gpu(p.sfb)
    d = _sentinel((p.G, p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_masked(_fp8(p.a), sfa, _fp8(p.b), sfb, torch.from_numpy(p.masked_m).cuda(), d)
    torch.cuda.synchronize()
    assert dg.get_device_error() == 0
    got = bits(d)
    valid_got, valid_ref = [], []
    for g, mg in enumerate(p.masked_m):
        assert (got[g, mg:] == SENTINEL).all(), f"expert {g}: masked rows were written"
        if mg == 0:
            continue
        ref = oracle_rows(p.a[g], sa[g], p.b[g], sb[g], p.M, p.N, p.K, np.arange(mg))
        check_close(got[g, :mg], ref, f"masked expert {g}")
        valid_got.append(got[g, :mg])
        valid_ref.append(ref)
    check_close(np.concatenate(valid_got), np.concatenate(valid_ref), "masked, all valid rows")
