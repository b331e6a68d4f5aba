"""GPU parity of the NN / TN / TT operand layouts (the ssnai.com analysis,
"SM90 vs SM100": SM100 serves NT, TN, NN and TT).  The oracle computes
D = A . B^T from A [M,K] and B [N,K]; the library receives the same bytes
stored K-major or MN-major as each layout prescribes, so the results must
agree exactly as for the NT layout."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close, packed

pytestmark = pytest.mark.gpu

# configurations built per layout: (block_n, ctas, pipes)
CONFIGS = {
    "tt": [(128, 1, 1), (224, 1, 1), (224, 2, 2)],  # A stored [K][M]
    "nn": [(128, 1, 1), (256, 1, 1), (256, 2, 1)],  # B stored [K][N]
    "tn": [(128, 1, 1), (256, 1, 1), (256, 2, 1)],  # both
}
CASES = [(layout, cfg) for layout, cfgs in CONFIGS.items() for cfg in cfgs]


@pytest.fixture(autouse=True)
def _clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.set_config(0)
    dg.get_device_error()
    yield
    dg.set_config(0)


def _stored(layout, a, b):
    """Device copies of the FP8 bytes of A [M,K] and B [N,K] in the layout's storage order."""
    a_s = np.ascontiguousarray(a.T) if layout[0] == "t" else a
    b_s = np.ascontiguousarray(b.T) if layout[1] == "n" else b
    to = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda().view(torch.float8_e4m3fn)
    return to(a_s), to(b_s)


def _run(layout, p, sa, sb):
    a, b = _stored(layout, p.a, p.b)
    d = dg.fp8_gemm(layout, a, torch.from_numpy(sa).cuda(), b, torch.from_numpy(sb).cuda())
    torch.cuda.synchronize()
    return bits(d)


@pytest.mark.parametrize("layout,cfg", CASES)
@pytest.mark.parametrize("shape", [(144, 384, 384), (400, 640, 640), (128, 512, 512)])
def test_layout_matches_oracle(layout, cfg, shape):
    M, N, K = shape
    p = synth.dense_problem(M, N, K, seed=91 + M)
    sa, sb = packed(p)
    dg.set_config(*cfg)
    got = _run(layout, p, sa, sb)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K)
    check_close(got, ref, f"{layout} {shape} cfg={cfg}")
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("layout,cfg", CASES)
def test_layout_integer_inputs_bit_exact(layout, cfg):
    """Small integers with unit scales: every product and sum is exact, so a
    misplaced element of an MN-major tile cannot hide inside the tolerance."""
    rng = np.random.default_rng(5)
    M, N, K = 256, 512, 384
    ai = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
    bi = rng.integers(-4, 5, size=(N, K)).astype(np.float32)
    a = torch.from_numpy(ai).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    b = torch.from_numpy(bi).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    p = synth.Problem("dense", "int", a, np.ones((M, K // 128), np.float32), b,
                      np.ones((N // 128, K // 128), np.float32), M, N, K)
    sa, sb = packed(p)
    dg.set_config(*cfg)
    got = _run(layout, p, sa, sb)
    assert np.array_equal(got, oracle.fp8_gemm_nt(a, sa, b, sb, M, N, K)), f"{layout} cfg={cfg}"


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_layout_heuristic_larger(layout):
    """The heuristic's own choice on a larger problem with per-block scales."""
    M, N, K = 1024, 1536, 1024
    p = synth.dense_problem(M, N, K, seed=95)
    sa, sb = packed(p)
    got = _run(layout, p, sa, sb)
    rows = np.arange(0, M, 7)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K, rows=rows)
    check_close(got[rows], ref, f"{layout} heuristic")
    assert dg.get_device_error() == 0


def test_layout_argument_errors():
    lib = dg.load()
    x = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    p = x.data_ptr()
    # A stored [K][M] needs M % 16 == 0 (16-byte row stride for TMA)
    assert lib.dg_fp8_gemm_tn(p, p, p, p, p, 24, 128, 128, None) == dg.DG_ERR_SHAPE
    assert lib.dg_fp8_gemm_tt(p, p, p, p, p, 24, 128, 128, None) == dg.DG_ERR_SHAPE
    assert lib.dg_fp8_gemm_nn(p, p, p, p, p, 16, 128, 100, None) == dg.DG_ERR_SHAPE
    assert lib.dg_fp8_gemm_nn(0, p, p, p, p, 16, 128, 128, None) == dg.DG_ERR_NULL
    with pytest.raises(ValueError):
        dg.fp8_gemm("xx", x, x, x, x)
