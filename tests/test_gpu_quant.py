"""GPU parity of the fused per-token FP8 quantisation (bit exact against the
oracle's hand-written E4M3 encoder and scale rule), and quantise -> GEMM."""
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
    dg.get_device_error()


def _special_input(shape, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape) * np.exp(rng.uniform(-12, 12, size=shape[:-1] + (1,)))
    flat = x.reshape(-1, shape[-1])
    flat[0, :128] = 0.0                                   # all-zero group
    if flat.shape[0] > 1:
        flat[1, :128] = 1e30 * np.sign(flat[1, :128])     # huge
    if flat.shape[0] > 2:
        flat[2, 128:256] *= 1e-35                         # tiny
    if flat.shape[0] > 3:
        flat[3, :128] = 448.0 * np.arange(128) / 127.0     # amax exactly 448
    return x


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(2, 37, 640), (1, 1, 128), (3, 5, 2048), (1, 4096, 2048)])
def test_quantize_bit_exact(dtype, shape):
    x = torch.from_numpy(_special_input(shape, seed=sum(shape))).to(dtype)
    q, sf = dg.quantize_fp8_1x128(x.cuda())
    torch.cuda.synchronize()
    codes, words = oracle.fp8_gemm.quantize_fp8_1x128(x.float().numpy().astype(np.float64))
    assert np.array_equal(q.view(torch.uint8).cpu().numpy(), codes)
    assert np.array_equal(sf.cpu().numpy(), words)
    assert dg.get_device_error() == 0


def test_quantize_then_gemm_matches_oracle():
    M, N, K = 300, 512, 1024
    x = torch.from_numpy(synth.normal(9, M * K).reshape(M, K)).to(torch.bfloat16)
    w = synth.dense_problem(8, N, K, seed=10)
    q, sf = dg.quantize_fp8_1x128(x.cuda())
    sb, _ = oracle.pack_sf_ue8m0(w.sfb[None])
    d = dg.fp8_gemm_nt(q, sf, torch.from_numpy(w.b).cuda().view(torch.float8_e4m3fn), torch.from_numpy(sb[0]).cuda())
    torch.cuda.synchronize()
    codes, words = oracle.fp8_gemm.quantize_fp8_1x128(x.float().numpy().astype(np.float64))
    ref = oracle.fp8_gemm_nt(codes, words, w.b, sb[0], M, N, K)
    check_close(bits(d), ref, "quantise -> gemm")
