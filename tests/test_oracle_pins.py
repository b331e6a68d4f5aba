"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources of truth used here: PyTorch's own float8_e4m3fn / bfloat16 conversions
(library routines), closed forms, exact rational (fractions.Fraction) brute
force, int64 arithmetic, the worked UE8M0 word of the scale-format reading,
and invariants of grouping and masking.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from moe_grouped_gemm_05_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _torch_e4m3(codes):
    t = torch.tensor(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.float().numpy().astype(np.float64)


def _torch_bf16_bits(x32):
    t = torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _e4m3_code(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


# ---------------------------------------------------------------- E4M3 / UE8M0


def test_e4m3_table_matches_torch_all_codes():
    tab = oracle.e4m3_table()
    ref = _torch_e4m3(np.arange(256))
    assert np.array_equal(np.isnan(tab), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(tab[ok], ref[ok])


def test_e4m3_spec_points():
    tab = oracle.e4m3_table()
    assert tab[0x38] == 1.0 and tab[0xB8] == -1.0
    assert tab[0x7E] == 448.0 and tab[0xFE] == -448.0   # largest finite
    assert tab[0x01] == 2.0 ** -9                        # smallest subnormal
    assert tab[0x07] == 7 * 2.0 ** -9                    # largest subnormal
    assert tab[0x08] == 2.0 ** -6                        # smallest normal
    assert np.isnan(tab[0x7F]) and np.isnan(tab[0xFF])   # the only NaNs
    assert np.isfinite(np.delete(tab, [0x7F, 0xFF])).all()  # no infinities


def test_ue8m0_worked_word():
    # exponents (127, 128, 126, 0) for K blocks 0..3 pack little-endian into 0x007E807F
    sf = np.array([[[1.0, 2.0, 0.5, 2.0 ** -127]]], dtype=np.float32)
    words, bad = oracle.pack_sf_ue8m0(sf)
    assert bad == 0
    assert words.shape == (1, 1, 4)
    assert words.view(np.uint32)[0, 0, 0] == 0x007E807F
    assert (words[0, 0, 1:] == 0).all()  # MN padding words are zero


def test_ue8m0_byte_is_log2_plus_127():
    k = np.arange(-126, 128)
    sf = np.ldexp(np.float32(1.0), k).astype(np.float32)
    byte, bad = oracle.ue8m0_from_f32(sf)
    _, ex = np.frexp(sf.astype(np.float64))  # library: sf = 0.5 * 2^ex
    assert not bad.any()
    assert np.array_equal(byte.astype(np.int64), (ex - 1) + 127)
    assert np.array_equal(oracle.ue8m0_value(byte), sf.astype(np.float64))
    assert oracle.ue8m0_value(np.array([0]))[0] == 2.0 ** -127
    assert np.isnan(oracle.ue8m0_value(np.array([255]))[0])


def test_ue8m0_rejects_non_powers_of_two():
    bad_vals = np.array([3.0, -1.0, 0.0, np.inf, -np.inf, np.nan, 2.0 ** -128, 1.5, -2.0 ** -127],
                        dtype=np.float32)
    byte, bad = oracle.ue8m0_from_f32(bad_vals)
    assert bad.all()
    assert (byte == 0).all()
    words, nbad = oracle.pack_sf_ue8m0(bad_vals.reshape(1, 1, -1))
    assert nbad == len(bad_vals)


def test_pack_unpack_round_trip_and_padding():
    rng = np.random.default_rng(7)
    batch, mn, kb = 3, 13, 7
    e = rng.integers(0, 255, size=(batch, mn, kb))
    sf = np.where(e == 0, np.float32(2.0 ** -127), np.ldexp(np.float32(1.0), e - 127)).astype(np.float32)
    words, bad = oracle.pack_sf_ue8m0(sf)
    assert bad == 0
    assert words.shape == (batch, 2, 16)
    back = oracle.unpack_sf_ue8m0(words, mn, kb)
    assert np.array_equal(back.astype(np.int64), e)
    w = words.view(np.uint32)
    assert (w[:, :, mn:] == 0).all()                 # MN padding
    assert (w[:, 1, :] >> 24 == 0).all()             # K block 7 does not exist: top byte 0
    # byte j of word [kp, m] is block 4*kp + j (spot check against the raw exponents)
    assert (w[1, 1, 5] >> 16) & 0xFF == e[1, 5, 6]
    assert w[2, 0, 12] & 0xFF == e[2, 12, 0]


# ---------------------------------------------------------------- BF16 rounding


def test_bf16_rne_matches_torch_on_float32_values():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(1000.0),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),       # BF16 subnormals
        (rng.standard_normal(2000) * 1e38).astype(np.float32),        # near overflow
        np.float32([0.0, -0.0, 1.0, 3.0e38, 3.4e38, -3.4e38]),
    ])
    # exact ties between neighbouring BF16 values
    base = rng.integers(0x0080, 0x7F00, size=4000).astype(np.uint32) << 16
    ties = (base | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    got = oracle.bf16_bits_from_f64(x.astype(np.float64))
    ref = _torch_bf16_bits(x)
    assert np.array_equal(got, ref)


def test_bf16_rne_rounds_once_from_double():
    # 1 + 2^-8 + 2^-40 is above the midpoint of [1, 1+2^-7]: rounds up.  Going
    # through float32 first would land on the midpoint and round to 1.0.
    x = np.array([1 + 2.0 ** -8 + 2.0 ** -40, 1 + 2.0 ** -8, -(1 + 3 * 2.0 ** -8), 2.0 ** -134 * 1.5,
                  (2 - 2.0 ** -8) * 2.0 ** 127])
    got = oracle.bf16_bits_from_f64(x)
    assert got[0] == 0x3F81
    assert got[1] == 0x3F80          # tie -> even
    assert got[2] == 0xBF82          # tie -> even (mantissa 2)
    assert got[3] == 0x0001          # 0.75 of the subnormal quantum 2^-133 rounds up to one quantum
    assert got[4] == 0x7F80          # tie at the top rounds to even = +inf


def _frac_to_bf16_bits(v: Fraction) -> int:
    """Exact-rational round to nearest even BF16 (independent of the oracle)."""
    if v == 0:
        return 0
    neg = v < 0
    a = -v if neg else v
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    qe = max(e, -126) - 7
    q = a / Fraction(2) ** qe
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = float(n * Fraction(2) ** qe)
    bits = int(np.float32(r).view(np.uint32)) >> 16
    return bits | (0x8000 if neg else 0)


def test_bf16_subnormal_quantum():
    x = np.array([2.0 ** -134 * 1.5, 2.0 ** -133 * 2.5, 2.0 ** -127])
    got = oracle.bf16_bits_from_f64(x)
    ref = [_frac_to_bf16_bits(Fraction(v)) for v in x]
    assert list(got) == ref


# ---------------------------------------------------------------- GEMM pins


def _pack(sf):
    w, bad = oracle.pack_sf_ue8m0(np.asarray(sf, np.float32)[None])
    assert bad == 0
    return w[0]


def test_all_ones_closed_form():
    M, N, K = 8, 256, 512
    a = np.full((M, K), 0x38, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    sfa = np.full((M, K // 128), 2.0 ** -3, np.float32)
    sfb = np.full((N // 128, K // 128), 2.0 ** 2, np.float32)
    d = oracle.fp8_gemm_nt(a, _pack(sfa), b, _pack(sfb), M, N, K)
    assert (d == 0x4380).all()  # K * 2^-3 * 2^2 = 256 exactly


def test_all_ones_per_block_scales():
    M, N, K = 4, 256, 512
    a = np.full((M, K), 0x38, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    ea = np.array([[127, 128, 126, 130]] * M)
    ea[1] = [120, 121, 122, 123]
    eb = np.array([[127, 127, 127, 127], [125, 129, 127, 126]])
    d = oracle.fp8_gemm_nt_f64(a, _pack(np.ldexp(1.0, ea - 127)), b, _pack(np.ldexp(1.0, eb - 127)), M, N, K)
    for m in range(M):
        for n in (0, 127, 128, 255):
            want = sum(128 * 2.0 ** (ea[m, k] - 127) * 2.0 ** (eb[n // 128, k] - 127) for k in range(4))
            assert d[m, n] == want


def test_small_integer_inputs_are_exact():
    rng = np.random.default_rng(3)
    M, N, K = 16, 384, 256
    ai = rng.integers(-4, 5, size=(M, K))
    bi = rng.integers(-4, 5, size=(N, K))
    a = _e4m3_code(ai.astype(np.float32))
    b = _e4m3_code(bi.astype(np.float32))
    assert np.array_equal(_torch_e4m3(a), ai)  # every integer in [-4, 4] is an E4M3 value
    ones_a = np.ones((M, K // 128), np.float32)
    ones_b = np.ones((3, K // 128), np.float32)
    d = oracle.fp8_gemm_nt(a, _pack(ones_a), b, _pack(ones_b), M, N, K)
    exact = ai.astype(np.int64) @ bi.astype(np.int64).T
    assert np.abs(exact).max() < 2 ** 24
    ref = _torch_bf16_bits(exact.astype(np.float32))
    assert np.array_equal(d, ref)


def test_brute_force_fraction_tiny():
    rng = np.random.default_rng(5)
    M, N, K = 3, 256, 256
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    a = rng.choice(finite, size=(M, K)).astype(np.uint8)
    b = rng.choice(finite, size=(N, K)).astype(np.uint8)
    ea = rng.integers(118, 136, size=(M, 2))
    eb = rng.integers(118, 136, size=(2, 2))
    d = oracle.fp8_gemm_nt(a, _pack(np.ldexp(1.0, ea - 127)), b, _pack(np.ldexp(1.0, eb - 127)), M, N, K)
    av = [[Fraction(float(v)) for v in row] for row in _torch_e4m3(a)]
    bv = [[Fraction(float(v)) for v in row] for row in _torch_e4m3(b)]
    cols = list(range(0, N, 17)) + [127, 128, 255]
    for m in range(M):
        for n in cols:
            tot = Fraction(0)
            for kb in range(2):
                s = sum(av[m][k] * bv[n][k] for k in range(kb * 128, kb * 128 + 128))
                tot += s * Fraction(2) ** int(ea[m, kb] - 127) * Fraction(2) ** int(eb[n // 128, kb] - 127)
            assert d[m, n] == _frac_to_bf16_bits(tot), (m, n)


def test_block_partial_exact_in_int64():
    rng = np.random.default_rng(9)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    a = rng.choice(finite, size=(32, 128)).astype(np.uint8)
    b = rng.choice(finite, size=(64, 128)).astype(np.uint8)
    tab = oracle.e4m3_table()
    ia = np.round(tab[a] * 512).astype(np.int64)   # every E4M3 value is a multiple of 2^-9
    ib = np.round(tab[b] * 512).astype(np.int64)
    assert np.array_equal(ia / 512.0, tab[a])
    exact = ia @ ib.T                               # products scaled by 2^18, exact
    ones = np.ones((32, 1), np.float32)
    f64 = oracle.fp8_gemm_nt_f64(a, _pack(ones), b, _pack(np.ones((1, 1), np.float32)), 32, 64, 128)
    assert np.array_equal(f64 * 2.0 ** 18, exact.astype(np.float64))


def test_scale_linearity_per_row_block():
    p = synth.dense_problem(8, 256, 384, seed=21)
    sa, sb = _pack(p.sfa), _pack(p.sfb)
    d0 = oracle.fp8_gemm_nt_f64(p.a, sa, p.b, sb, p.M, p.N, p.K)
    sfa2 = p.sfa.copy()
    sfa2[3, 1] *= 2
    d1 = oracle.fp8_gemm_nt_f64(p.a, _pack(sfa2), p.b, sb, p.M, p.N, p.K)
    assert np.array_equal(np.delete(d1, 3, 0), np.delete(d0, 3, 0))
    tab = oracle.e4m3_table()
    blk = tab[p.a[3, 128:256]] @ tab[p.b[:, 128:256]].T * p.sfa[3, 1] * np.repeat(p.sfb[:, 1], 128)[: p.N]
    assert np.allclose(d1[3] - d0[3], blk, rtol=1e-12, atol=0)


# ---------------------------------------------------------------- grouping pins


def test_contiguous_equals_per_expert_dense_and_padding_untouched():
    p = synth.contiguous_problem(3, 256, 256, rows=0, seed=31, counts=[130, 0, 70])
    sa = _pack(p.sfa)
    sb, _ = oracle.pack_sf_ue8m0(p.sfb)
    d = np.full((p.M, p.N), 0xDEAD, np.uint16)
    bad = oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, sa, p.b, sb, p.m_indices, d, p.G, p.N, p.K)
    assert bad == 0
    assert p.M == 256 + 128
    for e in range(p.G):
        rows = np.nonzero(p.m_indices == e)[0]
        if len(rows):
            ref = oracle.fp8_gemm_nt(p.a[rows], _pack(p.sfa[rows]), p.b[e], sb[e], len(rows), p.N, p.K)
            assert np.array_equal(d[rows], ref)
    assert (d[p.m_indices < 0] == 0xDEAD).all()


def test_contiguous_row_permutation_invariance():
    p = synth.contiguous_problem(2, 128, 128, rows=0, seed=33, counts=[100, 28])
    sb, _ = oracle.pack_sf_ue8m0(p.sfb)
    d = np.zeros((p.M, p.N), np.uint16)
    oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, _pack(p.sfa), p.b, sb, p.m_indices, d, p.G, p.N, p.K)
    perm = np.random.default_rng(1).permutation(p.M)
    d2 = np.zeros_like(d)
    oracle.m_grouped_fp8_gemm_nt_contiguous(p.a[perm], _pack(p.sfa[perm]), p.b, sb, p.m_indices[perm], d2,
                                            p.G, p.N, p.K)
    assert np.array_equal(d2, d[perm])


def test_masked_rows_untouched_and_clamped():
    p = synth.masked_problem(4, 256, 256, 256, seed=41, masked_m=[0, 256, 129, 7])
    sa, _ = oracle.pack_sf_ue8m0(p.sfa)
    sb, _ = oracle.pack_sf_ue8m0(p.sfb)
    d = np.full((p.G, p.M, p.N), 0xBEEF, np.uint16)
    bad = oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, p.masked_m, d, p.G, p.M, p.N, p.K)
    assert bad == 0
    for g, mg in enumerate(p.masked_m):
        assert (d[g, mg:] == 0xBEEF).all()
        if mg:
            ref = oracle.fp8_gemm_nt(p.a[g, :mg], _pack(p.sfa[g, :mg]), p.b[g], sb[g], mg, p.N, p.K)
            assert np.array_equal(d[g, :mg], ref)
    d3 = np.full((p.G, p.M, p.N), 0xBEEF, np.uint16)
    bad = oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, np.array([0, 300, -2, 7]), d3, p.G, p.M, p.N,
                                              p.K)
    assert bad == 2
    assert np.array_equal(d3[1], d[1]) and (d3[2] == 0xBEEF).all()


# ---------------------------------------------------------------- generator


def test_splitmix64_reference_value():
    # first output of SplitMix64 started from state 0 (Vigna's reference generator)
    assert int(synth.splitmix64(0, 0, 1)[0]) == 0xE220A8397B1DCDAF


def test_generator_is_deterministic_and_seeded():
    a1 = synth.dense_problem(64, 128, 256, seed=5)
    a2 = synth.dense_problem(64, 128, 256, seed=5)
    a3 = synth.dense_problem(64, 128, 256, seed=6)
    assert np.array_equal(a1.a, a2.a) and np.array_equal(a1.sfb, a2.sfb)
    assert not np.array_equal(a1.a, a3.a)


def test_quantisation_recipe_bounds():
    p = synth.dense_problem(32, 256, 512, seed=8)
    tab = oracle.e4m3_table()
    qa = tab[p.a]
    assert np.isfinite(qa).all() and np.abs(qa).max() <= 448
    # the scale is the smallest power of two that fits: the largest |x/s| of a group exceeds
    # 224, so its E4M3 rounding (spacing 32 there) is at least 224
    amax_q = np.abs(qa.reshape(32, 4, 128)).max(-1)
    assert (amax_q >= 224).all()


def test_zipf_routing_counts():
    c = synth.zipf_counts(1002 ^ 0x2121, 32768, 8, 1.1)
    assert c.sum() == 32768
    p = np.arange(1, 9) ** -1.1
    expect = 32768 * p / p.sum()
    assert np.all(np.abs(c - expect) < 5 * np.sqrt(expect))
    idx = synth.contiguous_indices(c)
    assert len(idx) % 128 == 0 and (idx >= 0).sum() == 32768


def test_topk_routing():
    """Top-1 routing by largest log-weight + Gumbel noise is a Zipf draw; top-k
    slots of a token are distinct experts; gates sum to one; the draw is seeded."""
    ids, g = synth.topk_routing(5, 40000, 1, 8, 1.1)
    c = np.bincount(ids[:, 0], minlength=8)
    p = np.arange(1, 9) ** -1.1
    expect = 40000 * p / p.sum()
    assert np.all(np.abs(c - expect) < 5 * np.sqrt(expect))
    ids2, g2 = synth.topk_routing(6, 5000, 3, 8, 1.1)
    assert ids2.shape == (5000, 3) and ids2.min() >= 0 and ids2.max() < 8
    assert all(len(set(r)) == 3 for r in ids2.tolist())
    assert np.allclose(g2.sum(axis=1), 1.0) and (g2 > 0).all()
    again, _ = synth.topk_routing(6, 5000, 3, 8, 1.1)
    assert np.array_equal(ids2, again)


def test_masked_counts_range():
    m = synth.uniform_masked_m(7, 1000, 256)
    assert m.min() >= 0 and m.max() <= 256 and 100 < m.mean() < 156


# ---------------------------------------------------------------- activation quantisation


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(12)
    y = np.concatenate([rng.standard_normal(50000) * 100, rng.standard_normal(5000) * 1e-3,
                        rng.uniform(-448, 448, 20000)])
    # exact midpoints between neighbouring E4M3 values (ties to even)
    tab = oracle.e4m3_table()
    pos = np.sort(tab[(np.arange(256) < 0x7F)])
    mids = (pos[1:] + pos[:-1]) / 2
    y = np.concatenate([y, mids, -mids, [0.0, -0.0, 448.0, -448.0]])
    y = np.clip(y.astype(np.float32).astype(np.float64), -448, 448)
    got = oracle.fp8_gemm.e4m3_encode_rne(y)
    ref = torch.from_numpy(y.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)
    assert oracle.fp8_gemm.e4m3_encode_rne(np.array([1000.0]))[0] == 0x7E  # saturates


def test_pow2_scale_is_smallest_fitting_power_of_two():
    f = oracle.fp8_gemm.pow2_scale_for_amax
    assert f(np.array([448.0]))[0] == 1.0 and f(np.array([449.0]))[0] == 2.0
    assert f(np.array([0.0]))[0] == 1.0
    one75 = np.float32(1.75)
    nxt = np.nextafter(one75, np.float32(2))
    assert f(np.array([float(one75)]))[0] == 2.0 ** -8
    assert f(np.array([float(nxt)]))[0] == 2.0 ** -7
    rng = np.random.default_rng(13)
    a = np.abs(rng.standard_normal(10000) * np.exp(rng.uniform(-40, 40, 10000)))
    s = f(a)
    assert np.all(a / s <= 448) and np.all(a / (s / 2) > 448)
    assert f(np.array([1e-45]))[0] == 2.0 ** -127   # clamped to the UE8M0 range


def test_quantize_worked_example():
    x = np.zeros((2, 128))
    x[0, 0], x[0, 5] = 448.0, -1.0
    x[1, 0], x[1, 1] = 449.0, 1e-3
    codes, words = oracle.fp8_gemm.quantize_fp8_1x128(x)
    assert codes[0, 0] == 0x7E and codes[0, 5] == 0xB8
    assert codes[1, 0] == 0x76  # 449 / 2 = 224.5 -> 224 (1.75 * 2^7)
    w = words.view(np.uint32)
    assert w[0, 0] == 127 and w[0, 1] == 128 and w[0, 2] == 0  # scales 1, 2; padding row


def test_quantize_agrees_with_the_generator_recipe():
    # the generator quantises with PyTorch's own cast; the oracle encodes by hand
    x = synth.normal(77, 5 * 384).reshape(5, 384)
    x[2] *= 1e-3
    x[3, :128] = 0.0
    q_gen, s_gen = synth.quantize_rows(x)
    codes, words = oracle.fp8_gemm.quantize_fp8_1x128(x)
    assert np.array_equal(codes, q_gen)
    assert np.array_equal(words, oracle.pack_sf_ue8m0(s_gen[None])[0][0])


# ---------------------------------------------------------------- 1D1D recipe, C accumulation


def test_1d1d_all_ones_closed_form_and_block_equivalence():
    M, N, K = 4, 256, 512
    a = np.full((M, K), 0x38, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    rng = np.random.default_rng(14)
    ea = rng.integers(124, 131, size=(M, 4))
    eb_row = rng.integers(124, 131, size=(N, 4))
    g = oracle.fp8_gemm.fp8_gemm_nt_general_f64
    d = g(a, _pack(np.ldexp(1.0, ea - 127)), b, _pack(np.ldexp(1.0, eb_row - 127)), M, N, K, sfb_gran_n=1)
    for m in range(M):
        for n in (0, 5, 129, 255):
            assert d[m, n] == sum(128 * 2.0 ** (ea[m, k] - 127) * 2.0 ** (eb_row[n, k] - 127) for k in range(4))
    # per-row scales that are constant over 128-row blocks reproduce the block recipe
    p = synth.dense_problem(8, 384, 256, seed=15)
    sa = _pack(p.sfa)
    per_row = np.repeat(p.sfb, 128, axis=0)[: p.N]
    d_row = g(p.a, sa, p.b, _pack(per_row), p.M, p.N, p.K, sfb_gran_n=1)
    d_blk = g(p.a, sa, p.b, _pack(p.sfb), p.M, p.N, p.K, sfb_gran_n=128)
    assert np.array_equal(d_row, d_blk)


def test_1d1d_brute_force_fraction():
    rng = np.random.default_rng(16)
    M, N, K = 2, 40, 256
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    a = rng.choice(finite, size=(M, K)).astype(np.uint8)
    b = rng.choice(finite, size=(N, K)).astype(np.uint8)
    ea = rng.integers(120, 134, size=(M, 2))
    eb = rng.integers(120, 134, size=(N, 2))
    d = oracle.fp8_gemm.fp8_gemm_nt_general_f64(a, _pack(np.ldexp(1.0, ea - 127)), b, _pack(np.ldexp(1.0, eb - 127)),
                                                 M, N, K, sfb_gran_n=1)
    av, bv = _torch_e4m3(a), _torch_e4m3(b)
    for m in range(M):
        for n in range(0, N, 7):
            tot = Fraction(0)
            for kb in range(2):
                s = sum(Fraction(float(av[m, k])) * Fraction(float(bv[n, k])) for k in range(kb * 128, kb * 128 + 128))
                tot += s * Fraction(2) ** int(ea[m, kb] - 127) * Fraction(2) ** int(eb[n, kb] - 127)
            assert Fraction(d[m, n]) == tot  # every term is exact in float64 here


def test_c_accumulation_adds_exactly():
    p = synth.dense_problem(8, 128, 256, seed=17)
    sa, sb = _pack(p.sfa), _pack(p.sfb)
    c = synth.normal(18, p.M * p.N).reshape(p.M, p.N)
    g = oracle.fp8_gemm.fp8_gemm_nt_general_f64
    d0 = g(p.a, sa, p.b, sb, p.M, p.N, p.K)
    d1 = g(p.a, sa, p.b, sb, p.M, p.N, p.K, c=c)
    assert np.allclose(d1 - d0, c.astype(np.float64), rtol=0, atol=1e-9 * np.abs(d0).max())
    assert np.array_equal(oracle.fp8_gemm.f32_bits_from_f64(np.array([1 + 2.0 ** -24, 1 + 3 * 2.0 ** -24])),
                          np.array([0x3F800000, 0x3F800002], np.uint32))  # ties to even


# ---------------------------------------------------------------- MoE permute / combine


def test_moe_permute_hand_example():
    ids = np.array([[1, 0], [2, -1], [1, 2], [0, 0]])
    m, row_of, src, Mt, bad = oracle.fp8_gemm.moe_permute(ids, 3, align=4)
    assert list(m) == [0, 0, 0, -1, 1, 1, -1, -1, 2, 2, -1, -1]
    assert row_of.tolist() == [[4, 0], [8, -1], [5, 9], [1, 2]]
    assert list(src) == [0, 3, 3, -1, 0, 2, -1, -1, 1, 2, -1, -1]
    assert Mt == 12 and bad == 0


def test_moe_permute_invariants():
    rng = np.random.default_rng(19)
    T, topk, G = 500, 3, 7
    check_permute_invariants(rng.integers(-1, G, size=(T, topk)), G)


def check_permute_invariants(ids, G):
    """What any correct contiguous-layout permutation of `ids` satisfies."""
    T, topk = ids.shape
    m, row_of, src, Mt, bad = oracle.fp8_gemm.moe_permute(ids, G)
    assert Mt % 128 == 0 and len(m) == Mt and bad == 0
    assert Mt <= oracle.fp8_gemm.moe_permute_capacity(T, topk, G)
    routed = ids >= 0
    rows = row_of[routed]
    assert len(set(rows.tolist())) == routed.sum()                 # each routed slot gets its own row
    assert np.array_equal(m[rows], ids[routed])                    # the row's expert is the slot's
    assert np.array_equal(src[rows], np.nonzero(routed)[0])        # ... and its source token
    assert (row_of[~routed] == -1).all() and ((m == -1) == (src == -1)).all()
    assert (np.diff(m[m >= 0]) >= 0).all()                         # expert segments in order
    for e in range(G):
        seg = np.nonzero(m == e)[0]
        if len(seg):
            assert seg[0] % 128 == 0 and (np.diff(seg) == 1).all()  # aligned, contiguous
            assert (np.diff(src[seg]) >= 0).all()                   # stable token order


def test_moe_combine_gathers_and_weights():
    rng = np.random.default_rng(20)
    D = oracle.bf16_bits_from_f64(rng.integers(-64, 64, size=(16, 32)).astype(np.float64))
    row_of = np.array([[3, -1], [0, 5], [7, 7]])
    out = oracle.fp8_gemm.moe_unpermute_combine(D, row_of)
    Dv = oracle.bf16_bits_to_f64(D)
    assert np.array_equal(oracle.bf16_bits_to_f64(out[0]), Dv[3])
    assert np.array_equal(oracle.bf16_bits_to_f64(out[1]), Dv[0] + Dv[5])   # small integers: exact
    w = np.array([[1.0, 0.0], [0.5, 0.25], [2.0, -1.0]], np.float32)
    out = oracle.fp8_gemm.moe_unpermute_combine(D, row_of, w)
    assert np.array_equal(oracle.bf16_bits_to_f64(out[2]), Dv[7])
