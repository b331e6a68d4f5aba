"""Edge cases at the boundaries of the entry points: empty problems, the
largest masked group count, narrow N, deep K, many small experts."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close, oracle_rows, packed, to_device

pytestmark = pytest.mark.gpu
SENTINEL = 0xDEAD


@pytest.fixture(autouse=True)
def _clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.set_config(0)
    dg.get_device_error()
    yield
    dg.set_config(0)


def _sentinel(shape):
    return torch.from_numpy(np.full(shape, SENTINEL, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def test_empty_problems_are_no_ops():
    lib = dg.load()
    x = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    p = x.data_ptr()
    assert lib.dg_fp8_gemm_nt(p, p, p, p, p, 0, 128, 128, None) == 0
    assert lib.dg_m_grouped_fp8_gemm_nt_contiguous(p, p, p, p, p, p, 0, 128, 128, 4, None) == 0
    assert lib.dg_m_grouped_fp8_gemm_nt_masked(p, p, p, p, p, p, 3, 0, 128, 128, None) == 0
    torch.cuda.synchronize()
    assert x.sum().item() == 0
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("N", [16, 48, 240])
def test_narrow_n(N):
    """N below one tile and not a multiple of 32: the epilogue clips its stores."""
    M, K = 200, 512
    p = synth.dense_problem(M, N, K, seed=500 + N)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    d = _sentinel((M, N))
    dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"], d)
    check_close(bits(d), oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K), f"N={N}")


def test_deep_k():
    """K = 16384: 128 K blocks, 32 scale words per row, long accumulation."""
    M, N, K = 130, 256, 16384
    p = synth.dense_problem(M, N, K, seed=501)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    for cfg in [(0, 0, 0), (128, 1, 1), (64, 1, 2)]:
        dg.set_config(*cfg)
        got = bits(dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"]))
        check_close(got, oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K), f"deep K cfg={cfg}")
    assert dg.get_device_error() == 0


def test_masked_largest_group_count():
    """512 experts (the masked layout's limit), most of them empty."""
    G, M_max, N, K = 512, 128, 128, 256
    rng = np.random.default_rng(502)
    mm = np.where(rng.random(G) < 0.1, rng.integers(1, M_max + 1, G), 0).astype(np.int32)
    mm[0], mm[-1] = M_max, 1
    p = synth.masked_problem(G, M_max, N, K, seed=502, masked_m=mm)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    d = _sentinel((G, M_max, N))
    dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], t["masked_m"], d)
    got = bits(d)
    ref = np.full((G, M_max, N), SENTINEL, np.uint16)
    oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, p.masked_m, ref, G, M_max, N, K)
    for g in range(G):
        m = int(mm[g])
        if m:
            check_close(got[g, :m], ref[g, :m], f"expert {g}")
        assert (got[g, m:] == SENTINEL).all()
    assert dg.get_device_error() == 0
    lib = dg.load()
    assert lib.dg_m_grouped_fp8_gemm_nt_masked(t["a"].data_ptr(), t["sfa"].data_ptr(), t["b"].data_ptr(),
                                               t["sfb"].data_ptr(), d.data_ptr(), t["masked_m"].data_ptr(),
                                               513, M_max, N, K, None) == dg.DG_ERR_SHAPE


def test_contiguous_many_small_experts():
    """64 experts with 0-200 rows each: many short segments, empty experts, and
    runs of one or two blocks (half-empty CTA pairs on the 2-CTA tiles)."""
    rng = np.random.default_rng(503)
    counts = rng.integers(0, 201, 64)
    p = synth.contiguous_problem(64, 256, 384, rows=0, seed=503, counts=list(counts))
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    ref = np.full((p.M, p.N), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, sa, p.b, sb, p.m_indices, ref, p.G, p.N, p.K) == 0
    valid = p.m_indices >= 0
    for cfg in [(0, 0, 0), (128, 1, 1), (224, 2, 2)]:
        dg.set_config(*cfg)
        d = _sentinel((p.M, p.N))
        dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"], d)
        got = bits(d)
        check_close(got[valid], ref[valid], f"many experts cfg={cfg}")
        assert (got[~valid] == SENTINEL).all()
    assert dg.get_device_error() == 0


def test_contiguous_pair_table_at_its_maximum():
    """1024 blocks of 128 rows (131072 rows, the most the 2-CTA tiles' pair
    table holds), 32 experts of 32 blocks each with ragged last blocks."""
    rng = np.random.default_rng(504)
    counts = 32 * 128 - rng.integers(0, 128, 32)
    p = synth.contiguous_problem(32, 256, 128, rows=0, seed=504, counts=list(counts))
    assert p.M == 1024 * 128
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    valid = p.m_indices >= 0
    ref = np.full((p.M, p.N), SENTINEL, np.uint16)
    for e in range(p.G):
        rows = np.nonzero(p.m_indices == e)[0]
        ref[rows] = oracle_rows(p.a, sa, p.b[e], sb[e], p.M, p.N, p.K, rows)
    dg.set_config(224, 2, 2)
    assert "(2cta)" in dg.describe_config("contiguous", p.M, p.N, p.K, p.G)
    d = _sentinel((p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"], d)
    got = bits(d)
    check_close(got[valid], ref[valid], "pair table with 1024 blocks")
    assert (got[~valid] == SENTINEL).all()
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("cfg", [(0, 0, 0), (224, 2, 2)])
def test_contiguous_all_padding_writes_nothing(cfg):
    p = synth.contiguous_problem(3, 256, 256, rows=0, seed=505, counts=[128, 128, 128])
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    t["m_indices"] = torch.full((p.M,), -1, dtype=torch.int32, device="cuda")
    dg.set_config(*cfg)
    d = _sentinel((p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"], d)
    assert (bits(d) == SENTINEL).all()
    assert dg.get_device_error() == 0
