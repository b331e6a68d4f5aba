"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on
the same seeded bytes.  Small problems are compared element by element;
scale packing, expert indexing and untouched rows bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import binding as dg
from moe_grouped_gemm_05_b200 import synth

from helpers import bits, check_close, packed, to_device

pytestmark = pytest.mark.gpu

# (block_n, ctas, pipes)
# (64|128, 1, 2) are the split-K tiles: both pipelines on every tile, each on half of K
BUILT = [(128, 1, 1), (224, 1, 1), (256, 1, 1), (128, 2, 1), (224, 2, 1), (256, 2, 1), (224, 2, 2), (128, 2, 2),
         (64, 1, 1), (64, 1, 2), (128, 1, 2)]
BUILT_1CTA = [c for c in BUILT if c[1] == 1 and c[2] == 1]
BUILT_CONTIG = [(128, 1, 1), (224, 1, 1), (256, 1, 1), (224, 2, 2)]  # the contiguous layout's configurations
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


# ------------------------------------------------------------------ packing


def test_pack_sf_bit_exact():
    rng = np.random.default_rng(1)
    e = rng.integers(1, 255, size=(3, 301, 17))
    sf = np.ldexp(np.float32(1.0), e - 127).astype(np.float32)
    sf[0, 0, 0] = 2.0 ** -127
    ref, bad = oracle.pack_sf_ue8m0(sf)
    assert bad == 0
    got = dg.pack_sf_ue8m0(torch.from_numpy(sf).cuda())
    assert dg.get_device_error() == 0
    assert np.array_equal(got.cpu().numpy(), ref)
    # 2-D input, kb multiple of 4, mn multiple of 4
    sf2 = np.ldexp(np.float32(1.0), rng.integers(100, 150, size=(56, 16)) - 127).astype(np.float32)
    ref2, _ = oracle.pack_sf_ue8m0(sf2[None])
    assert np.array_equal(dg.pack_sf_ue8m0(torch.from_numpy(sf2).cuda()).cpu().numpy(), ref2[0])


def test_pack_sf_rejects_bad_scales():
    sf = np.ones((1, 8, 8), np.float32)
    sf[0, 3, 5] = 3.0
    sf[0, 7, 0] = -0.5
    ref, bad = oracle.pack_sf_ue8m0(sf)
    assert bad == 2
    got = dg.pack_sf_ue8m0(torch.from_numpy(sf).cuda())
    assert dg.get_device_error() & dg.DG_DEVERR_BAD_SCALE
    assert np.array_equal(got.cpu().numpy(), ref)


# ------------------------------------------------------------------ dense


def _run_dense(p, sa=None, sb=None):
    t = to_device(p, sa, sb)
    d = dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"])
    torch.cuda.synchronize()
    return bits(d)


@pytest.mark.parametrize("cfg", BUILT)
def test_dense_small_all_configs(cfg):
    p = synth.WORKLOADS["dense_128x512x512"]()
    sa, sb = packed(p)
    dg.set_config(*cfg)
    got = _run_dense(p, sa, sb)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, p.M, p.N, p.K)
    check_close(got, ref, f"dense 128x512x512 cfg={cfg}")
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("cfg", BUILT)
@pytest.mark.parametrize("shape", [(200, 336, 384), (1, 16, 128), (129, 272, 640), (300, 1008, 1152),
                                   (520, 448, 256)])
def test_dense_ragged(cfg, shape):
    M, N, K = shape
    p = synth.dense_problem(M, N, K, seed=M * 7 + N + K)
    sa, sb = packed(p)
    dg.set_config(*cfg)
    got = _run_dense(p, sa, sb)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K)
    check_close(got, ref, f"dense {shape} cfg={cfg}")


def test_dense_integer_inputs_bit_exact():
    rng = np.random.default_rng(3)
    M, N, K = 256, 512, 512
    ai = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
    bi = rng.integers(-4, 5, size=(N, K)).astype(np.float32)
    a = torch.from_numpy(ai).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    b = torch.from_numpy(bi).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    p = synth.Problem("dense", "int", a, np.ones((M, K // 128), np.float32), b,
                      np.ones((N // 128, K // 128), np.float32), M, N, K)
    sa, sb = packed(p)
    for cfg in BUILT:
        dg.set_config(*cfg)
        got = _run_dense(p, sa, sb)
        ref = oracle.fp8_gemm_nt(a, sa, b, sb, M, N, K)
        assert np.array_equal(got, ref), f"cfg={cfg}"


def test_dense_all_ones_closed_form():
    M, N, K = 128, 256, 1024
    a = np.full((M, K), 0x38, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    sfa = np.full((M, K // 128), 2.0 ** -3, np.float32)
    sfb = np.full((N // 128, K // 128), 2.0 ** 2, np.float32)
    p = synth.Problem("dense", "ones", a, sfa, b, sfb, M, N, K)
    got = _run_dense(p)
    assert (got == 0x4400).all()  # 1024 * 2^-3 * 2^2 = 512


@pytest.mark.parametrize("cfg", BUILT)
@pytest.mark.parametrize("lo,hi,exact", [(124, 131, True), (112, 143, False)])
def test_dense_per_block_scales(cfg, lo, hi, exact):
    # all-ones operands, scales varying per row / per K block / per 128-column block.
    # With exponents in [124, 130] every block term is 128 * 2^[-6, 6] and the FP32
    # sum of eight of them is exact, so the result must match bit for bit; a wide
    # exponent range makes FP32 accumulation round, so only the tolerance applies.
    M, N, K = 256, 384, 1024
    rng = np.random.default_rng(4)
    ea = rng.integers(lo, hi, size=(M, K // 128))
    eb = rng.integers(lo, hi, size=(3, K // 128))
    p = synth.Problem("dense", "blk", np.full((M, K), 0x38, np.uint8), np.ldexp(1.0, ea - 127).astype(np.float32),
                      np.full((N, K), 0x38, np.uint8), np.ldexp(1.0, eb - 127).astype(np.float32), M, N, K)
    sa, sb = packed(p)
    dg.set_config(*cfg)
    got = _run_dense(p, sa, sb)
    ref = oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K)
    if exact:
        assert np.array_equal(got, ref)
    else:
        check_close(got, ref, "wide-range block scales")


# ------------------------------------------------------------------ contiguous


@pytest.mark.parametrize("cfg", BUILT_CONTIG)
def test_contiguous_small(cfg):
    p = synth.contiguous_problem(4, 512, 512, rows=0, seed=77, counts=[130, 0, 70, 250])
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    dg.set_config(*cfg)
    d = _sentinel((p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"], d)
    got = bits(d)
    ref = np.full((p.M, p.N), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, sa, p.b, sb, p.m_indices, ref, p.G, p.N, p.K) == 0
    valid = p.m_indices >= 0
    check_close(got[valid], ref[valid], f"contiguous cfg={cfg}")
    assert (got[~valid] == SENTINEL).all()
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("cfg", BUILT_CONTIG)
def test_contiguous_block_pairs_edge_layouts(cfg):
    """Blocks of one pair with different experts, an all-padding block first in
    a pair, a partly padded block, an expert repeated out of order and an odd
    number of blocks: every valid row matches the oracle, no other row is written."""
    layout = [(1, 128), (1, 60), (-1, 0), (0, 100), (2, 128), (2, 10), (0, 128)]  # (expert, rows) per block
    m_idx = np.full(128 * len(layout), -1, np.int32)
    for blk, (e, n) in enumerate(layout):
        m_idx[128 * blk:128 * blk + n] = e
    base = synth.contiguous_problem(3, 384, 384, rows=0, seed=78, counts=[128] * 7)
    p = synth.Problem("contiguous", "pairs", base.a, base.sfa, base.b, base.sfb, len(m_idx), base.N, base.K, 3,
                      m_indices=m_idx)
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    dg.set_config(*cfg)
    d = _sentinel((p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"], d)
    got = bits(d)
    ref = np.full((p.M, p.N), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, sa, p.b, sb, p.m_indices, ref, p.G, p.N, p.K) == 0
    valid = p.m_indices >= 0
    check_close(got[valid], ref[valid], f"contiguous pairs cfg={cfg}")
    assert (got[~valid] == SENTINEL).all()
    assert dg.get_device_error() == 0


@pytest.mark.parametrize("cfg", BUILT_CONTIG)
def test_contiguous_bad_expert_index_flags_and_skips(cfg):
    dg.set_config(*cfg)
    p = synth.contiguous_problem(2, 256, 256, rows=0, seed=78, counts=[128, 100])
    sa, sb = packed(p)
    idx = p.m_indices.copy()
    idx[5] = 9          # out of range inside a valid tile: row not written
    idx[130] = -3       # invalid negative
    t = to_device(p, sa, sb)
    t["m_indices"] = torch.from_numpy(idx).cuda()
    d = _sentinel((p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["m_indices"], d)
    err = dg.get_device_error()
    assert err & dg.DG_DEVERR_BAD_EXPERT
    got = bits(d)
    assert (got[5] == SENTINEL).all() and (got[130] == SENTINEL).all()
    ref = np.full((p.M, p.N), SENTINEL, np.uint16)
    oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, sa, p.b, sb, np.where(np.isin(np.arange(p.M), [5, 130]), -1, idx),
                                            ref, p.G, p.N, p.K)
    check_close(got, ref, "contiguous with bad rows")


# ------------------------------------------------------------------ masked


@pytest.mark.parametrize("cfg", BUILT)
def test_masked_small(cfg):
    p = synth.masked_problem(5, 256, 384, 640, seed=91, masked_m=[0, 256, 129, 7, 128])
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    dg.set_config(*cfg)
    d = _sentinel((p.G, p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], t["masked_m"], d)
    got = bits(d)
    ref = np.full((p.G, p.M, p.N), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, p.masked_m, ref, p.G, p.M, p.N, p.K) == 0
    for g, mg in enumerate(p.masked_m):
        assert (got[g, mg:] == SENTINEL).all(), f"expert {g}: rows >= {mg} were written"
        check_close(got[g, :mg], ref[g, :mg], f"masked expert {g} cfg={cfg}")
    assert dg.get_device_error() == 0


def test_masked_out_of_range_counts_are_clamped_and_flagged():
    p = synth.masked_problem(3, 128, 256, 256, seed=92, masked_m=[300, -4, 5])
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    d = _sentinel((p.G, p.M, p.N))
    dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], t["masked_m"], d)
    assert dg.get_device_error() & dg.DG_DEVERR_BAD_MASKED_M
    got = bits(d)
    ref = np.full((p.G, p.M, p.N), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, p.masked_m, ref, p.G, p.M, p.N, p.K) == 2
    check_close(got[0], ref[0], "clamped expert 0")
    assert (got[1] == SENTINEL).all()
    check_close(got[2, :5], ref[2, :5], "expert 2")
    assert (got[2, 5:] == SENTINEL).all()


def test_masked_is_graph_capturable_with_changing_counts():
    p = synth.masked_problem(4, 256, 256, 512, seed=93, masked_m=[10, 0, 200, 256])
    sa, sb = packed(p)
    t = to_device(p, sa, sb)
    d = torch.zeros((p.G, p.M, p.N), dtype=torch.bfloat16, device="cuda")
    mm = t["masked_m"]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], mm, d)  # warm-up
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], mm, d)
    for counts in ([1, 2, 3, 4], [256, 256, 0, 129]):
        d.zero_()
        mm.copy_(torch.tensor(counts, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        got = bits(d)
        ref = np.zeros((p.G, p.M, p.N), np.uint16)
        oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, np.array(counts), ref, p.G, p.M, p.N, p.K)
        for gi, mg in enumerate(counts):
            check_close(got[gi, :mg], ref[gi, :mg], f"graph replay expert {gi}")
            assert (got[gi, mg:] == 0).all()


@pytest.mark.parametrize("cfg", [(224, 2, 2), (128, 2, 2)])
@pytest.mark.parametrize("K", [896, 1024, 2048])
def test_odd_tile_count_splits_last_tile(cfg, K):
    """With two pipelines a CTA whose tile count is odd splits its last tile
    over both pipelines (each half of K, summed in the epilogue).  A small
    grid (4 CTA pairs) gives every pair 3 tiles; K spans 2..4 scale groups,
    with a ragged second half at K = 896."""
    M, N = 512, 6 * cfg[0]
    p = synth.dense_problem(M, N, K, seed=400 + K)
    sa, sb = packed(p)
    prev = dg.set_num_sms(8)
    try:
        dg.set_config(*cfg)
        got = _run_dense(p, sa, sb)
    finally:
        dg.set_num_sms(prev)
    check_close(got, oracle.fp8_gemm_nt(p.a, sa, p.b, sb, M, N, K), f"odd tiles cfg={cfg} K={K}")
    assert dg.get_device_error() == 0
