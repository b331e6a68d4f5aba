"""The GEMMs with A's scales as fp32 powers of two, packed by the kernel's
scale producer (the packing step fused into the GEMM): bit-identical to the
packed-word path, and a scale that is not a power of two is flagged."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close, packed, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dg.set_config(0)
    dg.get_device_error()
    yield
    dg.set_config(0)


@pytest.mark.parametrize("cfg", [(0, 0, 0), (128, 1, 1), (224, 2, 2), (64, 1, 2)])
@pytest.mark.parametrize("shape", [(200, 640, 640), (64, 512, 2048), (520, 384, 1152)])
def test_dense_fp32_scales_equal_packed(cfg, shape):
    M, N, K = shape
    p = synth.dense_problem(M, N, K, seed=300 + M)
    # wide per-row, per-block exponents so a wrong byte shows
    rng = np.random.default_rng(M)
    p.sfa[:] = np.ldexp(1.0, rng.integers(-20, 20, size=p.sfa.shape)).astype(np.float32)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    dg.set_config(*cfg)
    d_packed = bits(dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"]))
    d_f32 = bits(dg.fp8_gemm_nt(t["a"], torch.from_numpy(p.sfa).cuda(), t["b"], t["sfb"]))
    assert np.array_equal(d_f32, d_packed)
    check_close(d_f32, oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K), f"fp32 sfa {shape} {cfg}")
    assert dg.get_device_error() == 0


def test_grouped_fp32_scales_equal_packed():
    pc = synth.contiguous_problem(4, 512, 640, rows=0, seed=301, counts=[130, 0, 70, 250])
    sa, sb = packed(pc)
    t = to_device(pc, sa, sb)
    for cfg in [(0, 0, 0), (224, 1, 1), (224, 2, 2)]:
        dg.set_config(*cfg)
        ref = bits(dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"]))
        got = bits(dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], torch.from_numpy(pc.sfa).cuda(), t["b"], t["sfb"],
                                                       t["m_indices"]))
        valid = pc.m_indices >= 0
        assert np.array_equal(got[valid], ref[valid]), cfg
    pm = synth.masked_problem(5, 192, 384, 1024, seed=302, masked_m=[100, 0, 192, 7, 129])
    sa, sb = packed(pm)
    t = to_device(pm, sa, sb)
    dg.set_config(0)
    ref = bits(dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], t["masked_m"]))
    got = bits(dg.m_grouped_fp8_gemm_nt_masked(t["a"], torch.from_numpy(pm.sfa).cuda(), t["b"], t["sfb"],
                                               t["masked_m"]))
    for g, mg in enumerate(pm.masked_m):
        assert np.array_equal(got[g, :mg], ref[g, :mg]), g
    assert dg.get_device_error() == 0


def test_fp32_scale_not_power_of_two_is_flagged():
    M, N, K = 128, 256, 512
    p = synth.dense_problem(M, N, K, seed=303)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    sf = torch.from_numpy(p.sfa).cuda()
    sf[5, 2] = 3.0
    dg.fp8_gemm_nt(t["a"], sf, t["b"], t["sfb"])
    assert dg.get_device_error() & dg.DG_DEVERR_BAD_SCALE
    with pytest.raises(ValueError):
        dg.fp8_gemm_nt(t["a"], sf[:, :2].contiguous(), t["b"], t["sfb"])
