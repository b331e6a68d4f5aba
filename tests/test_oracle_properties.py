"""Property-based pins of the CPU oracle (hypothesis, derandomised).

Each property compares the oracle with something other than itself: exact
rational arithmetic over PyTorch's own E4M3 decode, an exact-rational
round-to-nearest-even, and the pack/unpack round trip over random shapes.
"""
from fractions import Fraction

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from test_oracle_pins import _frac_to_bf16_bits, _torch_e4m3

FINITE_CODES = [c for c in range(256) if (c & 0x7F) != 0x7F]
SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


def _pack(exps):
    sf = np.ldexp(np.float32(1.0), np.asarray(exps, np.int64) - 127).astype(np.float32)
    w, bad = oracle.pack_sf_ue8m0(sf[None])
    assert bad == 0
    return w[0]


@st.composite
def gemm_cases(draw):
    M = draw(st.integers(1, 3))
    N = draw(st.sampled_from([2, 130, 257]))
    kb = draw(st.integers(1, 3))
    K = 128 * kb
    nb = (N + 127) // 128
    seed = draw(st.integers(0, 2 ** 32 - 1))
    rng = np.random.default_rng(seed)
    a = rng.choice(FINITE_CODES, size=(M, K)).astype(np.uint8)
    b = rng.choice(FINITE_CODES, size=(N, K)).astype(np.uint8)
    ea = draw(st.lists(st.lists(st.integers(100, 150), min_size=kb, max_size=kb), min_size=M, max_size=M))
    eb = draw(st.lists(st.lists(st.integers(100, 150), min_size=kb, max_size=kb), min_size=nb, max_size=nb))
    return M, N, K, a, b, np.array(ea), np.array(eb)


@SETTINGS
@given(gemm_cases())
def test_gemm_equals_exact_rational_sum(case):
    M, N, K, a, b, ea, eb = case
    d = oracle.fp8_gemm_nt(a, _pack(ea), b, _pack(eb), M, N, K)
    av = [[Fraction(float(v)) for v in row] for row in _torch_e4m3(a)]
    bv = [[Fraction(float(v)) for v in row] for row in _torch_e4m3(b)]
    cols = sorted({0, N - 1, min(128, N - 1)})
    for m in range(M):
        for n in cols:
            tot = Fraction(0)
            for kb in range(K // 128):
                s = sum(av[m][k] * bv[n][k] for k in range(128 * kb, 128 * kb + 128))
                tot += s * Fraction(2) ** int(ea[m, kb] - 127) * Fraction(2) ** int(eb[n // 128, kb] - 127)
            assert d[m, n] == _frac_to_bf16_bits(tot), (m, n)


@SETTINGS
@given(st.integers(1, 3), st.integers(1, 9), st.integers(1, 9), st.integers(0, 2 ** 32 - 1))
def test_pack_unpack_round_trip(batch, mn, kb, seed):
    e = np.random.default_rng(seed).integers(0, 255, size=(batch, mn, kb))
    sf = np.where(e == 0, np.float32(2.0 ** -127), np.ldexp(np.float32(1.0), e - 127)).astype(np.float32)
    words, bad = oracle.pack_sf_ue8m0(sf)
    assert bad == 0
    assert words.shape == (batch, (kb + 3) // 4, (mn + 3) // 4 * 4)
    assert np.array_equal(oracle.unpack_sf_ue8m0(words, mn, kb).astype(np.int64), e)
    w = words.view(np.uint32)
    assert (w[:, :, mn:] == 0).all()                       # MN padding words
    if kb % 4:
        assert (w[:, -1, :] >> np.uint32(8 * (kb % 4)) == 0).all()   # missing K blocks of the last word


@SETTINGS
@given(st.floats(min_value=-3.0e38, max_value=3.0e38, allow_nan=False, allow_subnormal=True))
def test_bf16_rounding_equals_exact_rational(x):
    got = int(oracle.bf16_bits_from_f64(np.array([x]))[0])
    want = _frac_to_bf16_bits(Fraction(x))
    if x == 0:
        assert got & 0x7FFF == 0
    else:
        assert got == want, (x, hex(got), hex(want))


@SETTINGS
@given(st.integers(0x0080, 0x7F7E), st.booleans(), st.integers(-1, 1), st.integers(30, 44))
def test_bf16_rounding_near_midpoints(bits, negative, side, depth):
    """Values at, or a hair above or below, the midpoint between two
    neighbouring BF16 values: the cases where one rounding and a rounding
    through float32 first disagree."""
    lo = float(np.array([bits << 16], np.uint32).view(np.float32)[0])
    hi = float(np.array([(bits + 1) << 16], np.uint32).view(np.float32)[0])
    mid = Fraction(lo) + (Fraction(hi) - Fraction(lo)) / 2
    x = mid + side * (Fraction(hi) - Fraction(lo)) / 2 ** depth
    x = -x if negative else x
    xf = float(x)
    assert Fraction(xf) == x                                  # exactly representable in float64
    assert int(oracle.bf16_bits_from_f64(np.array([xf]))[0]) == _frac_to_bf16_bits(x)


@SETTINGS
@given(st.integers(1, 4), st.integers(1, 3), st.integers(0, 2 ** 32 - 1), st.integers(-30, 30))
def test_quantize_scale_is_minimal_and_codes_match_torch_cast(rows, groups, seed, log_mag):
    """Per 128-wide group: the scale s is the smallest power of two with
    amax / s <= 448 (1 for an all-zero group), and the codes are PyTorch's own
    float8_e4m3fn cast of x / s."""
    import torch

    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, 128 * groups)) * np.exp2(log_mag + rng.integers(-8, 9, size=(rows, 1)))
    x = x.astype(np.float32).astype(np.float64)
    if rows > 1:
        x[1, :128] = 0.0                                        # an all-zero group
    codes, words = oracle.fp8_gemm.quantize_fp8_1x128(x)
    e = oracle.unpack_sf_ue8m0(words[None], rows, groups)[0].astype(np.int64)
    for r in range(rows):
        for g in range(groups):
            grp = x[r, 128 * g:128 * (g + 1)]
            amax = Fraction(float(np.abs(grp).max()))
            s = Fraction(2) ** int(e[r, g] - 127)
            if amax == 0:
                assert s == 1
            else:
                assert amax / s <= 448 and amax / (s / 2) > 448
            ref = torch.from_numpy((grp / float(s)).astype(np.float32)).to(torch.float8_e4m3fn)
            assert np.array_equal(codes[r, 128 * g:128 * (g + 1)], ref.view(torch.uint8).numpy())


@SETTINGS
@given(st.integers(1, 300), st.integers(1, 4), st.integers(1, 40), st.floats(0.0, 0.5), st.integers(0, 2 ** 32 - 1))
def test_moe_permute_invariants_random(T, topk, G, drop, seed):
    from test_oracle_pins import check_permute_invariants

    rng = np.random.default_rng(seed)
    ids = rng.integers(0, G, size=(T, topk))
    ids[rng.random((T, topk)) < drop] = -1
    check_permute_invariants(ids, G)
