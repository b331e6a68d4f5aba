"""CPU oracle for the FP8 block-scaled GEMMs (test infrastructure only).

This is the plain, slow, obviously correct definition of what the GPU path
computes.  Only the test-suite, the package's smoke check and the benchmark's
CPU-baseline leg may import it; the product path never does.  It shares no
code with the CUDA library: it decodes every number format itself and uses
NumPy's float64 matmul only as the inner product of one 128-wide K block.

The operation (DeepGEMM pages, "细粒度缩放" / "两级累加结构" and the SF-format
notes under "UE8M0 int32 packing"):

    D[m, n] = bf16_rne( sum_kb  2^(ea[m,kb]-127) * 2^(eb[n//128,kb]-127)
                               * sum_{k in block kb} e4m3(a[m,k]) * e4m3(b[n,k]) )

where ea/eb are UE8M0 exponents unpacked from the int32 scale words.

Exactness.  Every E4M3 value is a multiple of 2^-9, so every product is a
multiple of 2^-18 and a 128-term block sum is bounded by 128*448^2 < 2^25:
each block partial fits in 43 significant bits and is exact in float64 in any
summation order, BLAS included.  Scaling by two powers of two is exact.  The
only roundings are the float64 sum over K blocks (<= K/128 terms, relative
error <= (K/128) * 2^-53) and the final round-to-nearest-even to BF16, done
directly from float64 (no intermediate float32, so no double rounding).

Parity pins: every function here is pinned in ``tests/test_oracle_pins.py``
against closed forms, PyTorch's own FP8/BF16 conversions, brute force in
exact rational arithmetic and integer arithmetic.
"""
from __future__ import annotations

import numpy as np

BLOCK = 128


# ---------------------------------------------------------------------------
# Number formats


def e4m3_table() -> np.ndarray:
    """Value of each of the 256 E4M3 ("E4M3FN") codes as float64.

    discosf.com DeepGEMM tutorial, section 2.3 (E4M3: 4 exponent and 3
    mantissa bits) and the float8_e4m3fn dtype of its section 4.2 example.
    Sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.  Exponent 0
    encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; there is no infinity, so
    the largest finite magnitude is 1.75 * 2^8 = 448.
    """
    codes = np.arange(256)
    s = np.where(codes & 0x80, -1.0, 1.0)
    e = (codes >> 3) & 0xF
    m = codes & 0x7
    sub = (m / 8.0) * 2.0 ** -6
    nor = (1.0 + m / 8.0) * np.ldexp(1.0, e - 7)
    v = s * np.where(e == 0, sub, nor)
    v[(codes & 0x7F) == 0x7F] = np.nan
    return v


def ue8m0_value(e: np.ndarray) -> np.ndarray:
    """2^(e-127) for UE8M0 exponent bytes (255 is NaN)."""
    e = np.asarray(e).astype(np.int64)
    v = np.ldexp(1.0, e - 127)
    return np.where(e == 255, np.nan, v)


def ue8m0_from_f32(sf: np.ndarray):
    """UE8M0 byte of each fp32 scale; returns (bytes, bad_mask).

    A valid scale is a positive finite power of two in the UE8M0 range:
    normal fp32 powers of two give their biased exponent field, and the
    subnormal 2^-127 gives 0.  Anything else is rejected (byte 0, bad=True).
    """
    bits = np.ascontiguousarray(sf, dtype=np.float32).view(np.uint32)
    sign = bits >> 31
    expf = (bits >> 23) & 0xFF
    mant = bits & 0x7FFFFF
    normal_ok = (sign == 0) & (expf >= 1) & (expf <= 254) & (mant == 0)
    sub127 = (sign == 0) & (expf == 0) & (mant == 0x400000)  # 2^-127 = 2^22 * 2^-149
    ok = normal_ok | sub127
    byte = np.where(normal_ok, expf, 0).astype(np.uint8)
    return byte, ~ok


def packed_sf_shape(mn: int, kb: int):
    """(words along K, words along MN) of one packed scale matrix."""
    return (kb + 3) // 4, (mn + 3) // 4 * 4


def pack_sf_ue8m0(sf: np.ndarray):
    """Pack fp32 power-of-two scales [batch, MN, Kb] into UE8M0 int32 words.

    Output int32 [batch, ceil(Kb/4), align4(MN)], MN contiguous ("transposed",
    MN-major).  Byte j (bits 8j..8j+7, little-endian) of word [kp, mn] holds
    the exponent of scale [mn, 4*kp + j].  Padding bytes (kb >= Kb, mn >= MN)
    are 0.  Returns (words, number of rejected scales).
    """
    sf = np.asarray(sf, dtype=np.float32)
    batch, mn, kb = sf.shape
    byte, bad = ue8m0_from_f32(sf)
    kp, mn4 = packed_sf_shape(mn, kb)
    buf = np.zeros((batch, mn4, kp * 4), dtype=np.uint32)
    buf[:, :mn, :kb] = byte
    words = np.zeros((batch, kp, mn4), dtype=np.uint32)
    for j in range(4):
        words |= buf[:, :, j::4].transpose(0, 2, 1) << np.uint32(8 * j)
    return words.view(np.int32), int(bad.sum())


def unpack_sf_ue8m0(words: np.ndarray, mn: int, kb: int) -> np.ndarray:
    """Inverse of :func:`pack_sf_ue8m0`: UE8M0 bytes [batch, MN, Kb]."""
    w = np.asarray(words).view(np.uint32)
    if w.ndim == 2:
        w = w[None]
    batch = w.shape[0]
    out = np.zeros((batch, mn, kb), dtype=np.uint8)
    for k in range(kb):
        out[:, :, k] = ((w[:, k // 4, :mn] >> np.uint32(8 * (k % 4))) & 0xFF).astype(np.uint8)
    return out


def bf16_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """Round float64 values to BF16 (round to nearest, ties to even); uint16 bits.

    BF16 keeps 8 significant bits; its normal range starts at 2^-126 and its
    subnormals are multiples of 2^-133.  For each x the quantum is
    2^(floor(log2|x|) - 7) (or 2^-133 below the normal range); x is divided by
    the quantum (exact: a power of two), rounded half-to-even to an integer
    and scaled back, which is exact.  Results of magnitude >= 2^128 overflow
    to infinity.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    fin = np.isfinite(x) & (x != 0)
    _, ex = np.frexp(np.where(fin, x, 1.0))
    lg = ex - 1  # floor(log2|x|)
    qexp = np.where(lg < -126, -133, lg - 7)
    q = np.rint(np.ldexp(np.where(fin, x, 0.0), -qexp))
    r = np.ldexp(q, qexp)
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, x), r)
    out[...] = np.where(fin, r, x)
    f32 = out.astype(np.float32)  # exact: every r is a BF16 value
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    bits = np.where(np.isnan(x), np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# GEMMs


def _decode(codes: np.ndarray) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, dtype=np.uint8)]


def fp8_gemm_nt_f64(a, sfa_words, b, sfb_words, M, N, K, rows=None, cols=None) -> np.ndarray:
    """Unrounded float64 D = A . B^T with per-128-K scale promotion.

    a: uint8 [M,K] E4M3; b: uint8 [N,K] E4M3; sfa_words: int32 packed scales of
    A (MN = M rows, one per 128 K); sfb_words: int32 packed scales of B (MN =
    ceil(N/128) blocks).  ``rows``/``cols`` select a sub-block of D.
    """
    Kb = K // BLOCK
    assert K % BLOCK == 0
    ea = unpack_sf_ue8m0(sfa_words, M, Kb)[0]
    eb = unpack_sf_ue8m0(sfb_words, (N + BLOCK - 1) // BLOCK, Kb)[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    cols = np.arange(N) if cols is None else np.asarray(cols)
    A = _decode(a[rows])
    B = _decode(b[cols])
    acc = np.zeros((len(rows), len(cols)), dtype=np.float64)
    for kb in range(Kb):
        ks = slice(kb * BLOCK, (kb + 1) * BLOCK)
        partial = A[:, ks] @ B[:, ks].T                  # exact (see module doc)
        sa = ue8m0_value(ea[rows, kb])                    # [rows]
        sb = ue8m0_value(eb[cols // BLOCK, kb])           # [cols]
        acc += partial * sa[:, None] * sb[None, :]        # two exact power-of-two scalings
    return acc


def fp8_gemm_nt(a, sfa_words, b, sfb_words, M, N, K, rows=None, cols=None) -> np.ndarray:
    """BF16 bits of D = A . B^T (dense NT layout, D row-major [M,N])."""
    return bf16_bits_from_f64(fp8_gemm_nt_f64(a, sfa_words, b, sfb_words, M, N, K, rows, cols))


def m_grouped_fp8_gemm_nt_contiguous(a, sfa_words, b, sfb_words, m_indices, d_bits, G, N, K):
    """Contiguous M-grouped GEMM, written into ``d_bits`` (uint16 [M_total,N]) in place.

    Row m with e = m_indices[m] >= 0 gets D[m] = A[m] . B[e]^T with A's row
    scales and expert e's block scales; rows with e == -1 are not written.
    Returns the number of rows with an out-of-range expert index (not written).
    """
    M_total = a.shape[0]
    bad = 0
    for e in range(G):
        rows = np.nonzero(m_indices == e)[0]
        if len(rows) == 0:
            continue
        d_bits[rows] = fp8_gemm_nt(a, sfa_words, b[e], sfb_words[e], M_total, N, K, rows=rows)
    bad += int(((m_indices < -1) | (m_indices >= G)).sum())
    return bad


def m_grouped_fp8_gemm_nt_masked(a, sfa_words, b, sfb_words, masked_m, d_bits, G, M_max, N, K):
    """Masked M-grouped GEMM, written into ``d_bits`` (uint16 [G,M_max,N]) in place.

    For each expert g, rows m < masked_m[g] get D[g,m] = A[g,m] . B[g]^T; rows
    m >= masked_m[g] are not written.  Counts outside [0, M_max] are clamped
    into it; the number of such counts is returned.
    """
    bad = 0
    for g in range(G):
        mg = int(masked_m[g])
        if mg < 0 or mg > M_max:
            bad += 1
            mg = min(max(mg, 0), M_max)
        if mg == 0:
            continue
        d_bits[g, :mg] = fp8_gemm_nt(a[g], sfa_words[g], b[g], sfb_words[g], M_max, N, K,
                                     rows=np.arange(mg))
    return bad


# ---------------------------------------------------------------------------
# Per-token 1x128 quantisation (the activation side of the recipe)


def e4m3_encode_rne(y: np.ndarray) -> np.ndarray:
    """E4M3FN codes of float64 values: round to nearest, ties to even, saturating at +-448.

    Negative inputs keep the sign bit even when they round to zero (-0 is 0x80).

    Normal values 2^-6 <= |y| have 3 mantissa bits, so their quantum is
    2^(floor(log2|y|) - 3); below 2^-6 the quantum is the subnormal step 2^-9.
    y is divided by its quantum (exact: a power of two), rounded half-to-even,
    scaled back and clamped to 448; the code is then built field by field.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    lg = ex - 1
    qexp = np.where(lg < -6, -9, lg - 3)
    v = np.ldexp(np.rint(np.ldexp(a, -qexp)), qexp)
    v = np.minimum(v, 448.0)
    # encode v (a representable magnitude) into exponent / mantissa fields
    _, ev = np.frexp(np.where(v > 0, v, 1.0))
    lv = ev - 1
    sub = v < 2.0 ** -6
    e_field = np.where(sub, 0, lv + 7)
    m_field = np.where(sub, np.rint(v / 2.0 ** -9), np.rint((v / np.ldexp(1.0, lv) - 1.0) * 8))
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = np.where(v == 0, 0, code)
    sign = np.signbit(y).astype(np.int64) << 7  # negative values keep their sign, -0 included
    return (code | sign).astype(np.uint8)


def pow2_scale_for_amax(amax: np.ndarray) -> np.ndarray:
    """Smallest power of two s with amax / s <= 448, within UE8M0's [2^-127, 2^127]; 1 for amax = 0."""
    amax = np.asarray(amax, dtype=np.float64)
    r = amax / 448.0  # only the comparison with powers of two matters: do it exactly below
    _, e = np.frexp(np.where(amax > 0, r, 1.0))
    c = e.astype(np.int64)  # r < 2^e; 2^(e-1) <= r
    exact_half = np.ldexp(448.0, e - 1) >= amax  # 448 * 2^(e-1) >= amax, decided exactly
    c = np.where(exact_half, e - 1, e)
    c = np.clip(c, -127, 127)
    return np.where(amax > 0, np.ldexp(1.0, c), 1.0)


def quantize_fp8_1x128(x: np.ndarray):
    """Quantises x[..., M, K] per row and 128-wide K group.

    Returns (E4M3 codes with x's shape, packed UE8M0 words [..., ceil(K/512), align4(M)]).
    The scale of a group is the smallest power of two s with max|x|/s <= 448.
    """
    x = np.asarray(x, dtype=np.float64)
    *lead, M, K = x.shape
    assert K % BLOCK == 0
    g = x.reshape(*lead, M, K // BLOCK, BLOCK)
    s = pow2_scale_for_amax(np.abs(g).max(axis=-1))
    codes = e4m3_encode_rne(g / s[..., None]).reshape(x.shape)
    sf = s.astype(np.float32)
    sf3 = sf.reshape(-1, M, K // BLOCK)
    words, bad = pack_sf_ue8m0(sf3)
    assert bad == 0
    return codes, words.reshape(*lead, *words.shape[1:])


def fp8_gemm_nt_general_f64(a, sfa_words, b, sfb_words, M, N, K, sfb_gran_n=128, c=None, rows=None):
    """D = A . B^T (+ C) with per-128-K promotion, unrounded float64.

    sfb_gran_n = 128: B carries one scale per 128x128 block ("1D2D", the
    default recipe); sfb_gran_n = 1: one scale per row of B and 128-wide K
    block ("1D1D"), packed with MN = N.  c, if given, is an fp32 [M, N]
    matrix added to the exact product before the output rounding.
    """
    Kb = K // BLOCK
    assert K % BLOCK == 0 and sfb_gran_n in (1, 128)
    ea = unpack_sf_ue8m0(sfa_words, M, Kb)[0]
    eb = unpack_sf_ue8m0(sfb_words, -(-N // sfb_gran_n), Kb)[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    A = _decode(a[rows])
    B = _decode(b)
    acc = np.zeros((len(rows), N), dtype=np.float64)
    cols = np.arange(N) // sfb_gran_n
    for kb in range(Kb):
        ks = slice(kb * BLOCK, (kb + 1) * BLOCK)
        acc += (A[:, ks] @ B[:, ks].T) * ue8m0_value(ea[rows, kb])[:, None] * ue8m0_value(eb[cols, kb])[None, :]
    if c is not None:
        acc += np.asarray(c, dtype=np.float32)[rows].astype(np.float64)
    return acc


def f32_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """Round float64 to float32 (IEEE round to nearest even, as NumPy's cast); uint32 bits."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32)


# ---------------------------------------------------------------------------
# MoE permutation into the contiguous layout, and the weighted combine


def moe_permute(topk_ids: np.ndarray, num_experts: int, align: int = BLOCK):
    """Contiguous-layout permutation of routed token slots (group_by_expert).

    topk_ids[t, s] is the expert of slot s of token t (-1: not routed).  Expert
    segments follow in expert order; inside a segment the slots keep their
    (token, slot) order; each segment is padded with -1 rows to a multiple of
    `align`.  Returns (m_indices [M_total], row_of [T, topk] with -1 for
    unrouted slots, src_of [M_total] with the source token of each row or -1,
    M_total, bad) where bad counts ids outside [-1, num_experts).
    """
    ids = np.asarray(topk_ids, dtype=np.int64)
    T, topk = ids.shape
    flat = ids.reshape(-1)
    bad = int(((flat < -1) | (flat >= num_experts)).sum())
    m_indices, src_of = [], []
    row_of = np.full(T * topk, -1, dtype=np.int64)
    row = 0
    for e in range(num_experts):
        slots = np.nonzero(flat == e)[0]          # ascending (token, slot) order
        row_of[slots] = row + np.arange(len(slots))
        padded = -(-len(slots) // align) * align
        m_indices += [e] * len(slots) + [-1] * (padded - len(slots))
        src_of += list(slots // topk) + [-1] * (padded - len(slots))
        row += padded
    return (np.array(m_indices, dtype=np.int32), row_of.reshape(T, topk).astype(np.int32),
            np.array(src_of, dtype=np.int32), row, bad)


def moe_permute_capacity(T: int, topk: int, num_experts: int, align: int = BLOCK) -> int:
    """Rows that always suffice for the contiguous layout: align(T*topk + (align-1)*num_experts)."""
    return -(-(T * topk + (align - 1) * num_experts) // align) * align


def moe_unpermute_combine(d_bits: np.ndarray, row_of: np.ndarray, weights=None) -> np.ndarray:
    """out[t] = bf16( sum_s w[t,s] * D[row_of[t,s]] ) over routed slots, summed in float64."""
    D = bf16_bits_to_f64(d_bits)
    T, topk = row_of.shape
    w = np.ones((T, topk)) if weights is None else np.asarray(weights, dtype=np.float32).astype(np.float64)
    out = np.zeros((T, D.shape[1]))
    for s in range(topk):
        r = row_of[:, s]
        ok = r >= 0
        out[ok] += w[ok, s][:, None] * D[r[ok]]
    return bf16_bits_from_f64(out)
