"""GPU parity of the extended dense entry point: the 1D1D recipe (per-row B
scales), FP32 output and accumulation into an FP32 C.

FP32 outputs keep the BF16 tolerance's row term: |x - y| <= ulp_f32(y) + 2^-10 * max|y[row]|,
with the normalised difference < 1e-4; integer-valued problems are bit exact."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.set_config(0)
    dg.get_device_error()
    yield
    dg.set_config(0)


def _check_f32(got, ref, what):
    x = got.astype(np.float64)
    y = ref.astype(np.float64)
    rowmax = np.abs(y).max(axis=1, keepdims=True)
    ulp = np.spacing(np.abs(y).astype(np.float32)).astype(np.float64)
    bad = np.abs(x - y) > ulp + 2.0 ** -10 * rowmax
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance"
    den = float((x * x + y * y).sum())
    assert den == 0 or 1.0 - 2.0 * float((x * y).sum()) / den < 1e-4


def _dev(p, sfb_words):
    sa, _ = oracle.pack_sf_ue8m0(p.sfa[None])
    return (torch.from_numpy(p.a).cuda().view(torch.float8_e4m3fn), torch.from_numpy(sa[0]).cuda(),
            torch.from_numpy(p.b).cuda().view(torch.float8_e4m3fn), torch.from_numpy(sfb_words).cuda(), sa[0])


def _row_scales(N, K, seed):
    rng = np.random.default_rng(seed)
    return np.ldexp(1.0, rng.integers(-10, 3, size=(N, K // 128))).astype(np.float32)


@pytest.mark.parametrize("cfg", [(128, 1), (224, 1), (256, 1), (224, 2), (224, 2, 2)])
@pytest.mark.parametrize("shape", [(200, 336, 384), (256, 512, 1024)])
def test_1d1d_bf16(cfg, shape):
    M, N, K = shape
    p = synth.dense_problem(M, N, K, seed=M + N)
    sf_row = _row_scales(N, K, seed=M)
    sb, _ = oracle.pack_sf_ue8m0(sf_row[None])
    a, sfa, b, sfb, sa = _dev(p, sb[0])
    dg.set_config(*cfg)
    d = dg.fp8_gemm_nt_ex(a, sfa, b, sfb, recipe_b=1)
    torch.cuda.synchronize()
    ref = oracle.bf16_bits_from_f64(oracle.fp8_gemm.fp8_gemm_nt_general_f64(p.a, sa, p.b, sb[0], M, N, K, sfb_gran_n=1))
    check_close(bits(d), ref, f"1d1d {shape} {cfg}")
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("recipe_b", [128, 1])
@pytest.mark.parametrize("with_c", [False, True])
@pytest.mark.parametrize("shape", [(200, 336, 384), (1, 16, 128), (4096, 7168, 2048)])
def test_fp32_output_and_c(recipe_b, with_c, shape):
    M, N, K = shape
    p = synth.dense_problem(M, N, K, seed=3 * M + N)
    sfb_src = p.sfb if recipe_b == 128 else _row_scales(N, K, seed=N)
    sb, _ = oracle.pack_sf_ue8m0(sfb_src[None])
    a, sfa, b, sfb, sa = _dev(p, sb[0])
    c = synth.normal(M + 1, M * N, sigma=10.0).reshape(M, N) if with_c else None
    d = dg.fp8_gemm_nt_ex(a, sfa, b, sfb, c=torch.from_numpy(c).cuda() if with_c else None, recipe_b=recipe_b,
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 512 else np.array([0, 1, 127, 128, 2048, 4095])
    ref = oracle.fp8_gemm.fp8_gemm_nt_general_f64(p.a, sa, p.b, sb[0], M, N, K, sfb_gran_n=recipe_b, c=c, rows=rows)
    _check_f32(d.cpu().numpy()[rows], ref.astype(np.float32), f"fp32 {shape} recipe {recipe_b} c={with_c}")
    assert dg.get_device_error() == 0


def test_fp32_integer_inputs_bit_exact():
    rng = np.random.default_rng(21)
    M, N, K = 256, 512, 512
    ai = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
    bi = rng.integers(-4, 5, size=(N, K)).astype(np.float32)
    a = torch.from_numpy(ai).to(torch.float8_e4m3fn)
    b = torch.from_numpy(bi).to(torch.float8_e4m3fn)
    ones_a, _ = oracle.pack_sf_ue8m0(np.ones((1, M, K // 128), np.float32))
    ones_b, _ = oracle.pack_sf_ue8m0(np.ones((1, N, K // 128), np.float32))
    c = rng.integers(-1000, 1000, size=(M, N)).astype(np.float32)
    d = dg.fp8_gemm_nt_ex(a.cuda(), torch.from_numpy(ones_a[0]).cuda(), b.cuda(), torch.from_numpy(ones_b[0]).cuda(),
                          c=torch.from_numpy(c).cuda(), recipe_b=1, out_dtype=torch.float32)
    exact = (ai.astype(np.int64) @ bi.astype(np.int64).T + c.astype(np.int64)).astype(np.float32)
    assert np.array_equal(d.cpu().numpy(), exact)


def test_ex_argument_errors():
    p = synth.dense_problem(128, 128, 128, seed=1)
    sb, _ = oracle.pack_sf_ue8m0(p.sfb[None])
    a, sfa, b, sfb, _ = _dev(p, sb[0])
    with pytest.raises(dg.DGError):
        dg.fp8_gemm_nt_ex(a, sfa, b, sfb, c=torch.zeros((128, 128), device="cuda"), out_dtype=torch.bfloat16)
