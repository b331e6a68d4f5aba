"""Decode-sized problems (at most 64 rows of A per group) on the split-K tiles
with 64-row A stages: the MMA stays 128 rows tall and its upper half reads
whatever lies in the next 8 KB of shared memory, so these tests check that
the valid rows equal the oracle's and that nothing beyond them is written."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close, packed, to_device

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


@pytest.mark.parametrize("M", [1, 17, 63, 64])
@pytest.mark.parametrize("K", [1536, 2048])
@pytest.mark.parametrize("cfg", [(0, 0, 0), (64, 1, 2)])
def test_dense_decode_rows(M, K, cfg):
    """Valid rows match the oracle; the rows after D (a larger buffer's tail) keep their sentinel."""
    N = 464  # seven 64-wide tiles and a ragged 16-column one
    p = synth.dense_problem(M, N, K, seed=900 + M + K)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    dg.set_config(*cfg)
    full = _sentinel((M + 64, N))
    dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"], full[:M])
    got = bits(full)
    check_close(got[:M], oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K), f"M={M} K={K} cfg={cfg}")
    assert (got[M:] == SENTINEL).all(), "rows beyond M were written"
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("cfg", [(0, 0, 0), (64, 1, 2)])
def test_masked_decode_rows(cfg):
    G, M_max, N, K = 4, 64, 256, 2048
    mm = np.array([64, 0, 17, 1], np.int32)
    p = synth.masked_problem(G, M_max, N, K, seed=910, masked_m=mm)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    dg.set_config(*cfg)
    d = _sentinel((G, M_max, N))
    dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], t["masked_m"], d)
    got = bits(d)
    ref = np.full((G, M_max, N), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, mm, ref, G, M_max, N, K) == 0
    for g in range(G):
        m = int(mm[g])
        if m:
            check_close(got[g, :m], ref[g, :m], f"expert {g} cfg={cfg}")
        assert (got[g, m:] == SENTINEL).all(), f"masked rows of expert {g} were written"
    assert dg.get_device_error() == 0
