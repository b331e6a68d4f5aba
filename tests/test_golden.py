"""The oracle against the hand-derived worked examples in ``tests/golden/``.

Each fixture states its source passage and shows its arithmetic; nothing in
them was produced by the oracle or by the CUDA path.
"""
from fractions import Fraction
from pathlib import Path

import numpy as np
import pytest

import oracle

GOLDEN = Path(__file__).parent / "golden"

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rows(name):
    """Non-comment lines of a fixture, split into fields; '[section]' lines kept."""
    out = []
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if line:
            out.append(line.split())
    return out


def _sections(name):
    sec, cur = {}, None
    for f in _rows(name):
        if f[0].startswith("["):
            cur = sec.setdefault(f[0].strip("[]"), [])
        else:
            cur.append(f)
    return sec


def test_e4m3_codes():
    tab = oracle.e4m3_table()
    rows = _rows("e4m3_codes.txt")
    assert len(rows) >= 20
    for code, val in rows:
        got = tab[int(code, 16)]
        if val == "nan":
            assert np.isnan(got), code
        elif val == "-0":
            assert got == 0 and np.signbit(got), code
        else:
            assert Fraction(got) == Fraction(val), (code, got, val)
            assert not (val == "0" and np.signbit(got))


def test_ue8m0_words():
    sec = _sections("ue8m0_words.txt")
    for f in sec["word"]:
        ks, want = f[:4], int(f[4], 16)
        ks = [k for k in ks if k != "-"]
        sf = np.ldexp(np.float32(1.0), np.array(ks, dtype=np.int64)).astype(np.float32)
        words, bad = oracle.pack_sf_ue8m0(sf.reshape(1, 1, -1))
        assert bad == 0
        assert words.view(np.uint32)[0, 0, 0] == want, (f, hex(words.view(np.uint32)[0, 0, 0]))
        assert (words[0, 0, 1:] == 0).all()
        back = oracle.unpack_sf_ue8m0(words, 1, len(ks))
        assert back[0, 0].tolist() == [int(k) + 127 for k in ks]

    mat = {f[0]: f[1:] for f in sec["matrix"] if f[0] in ("mn", "kb")}
    mn, kb = int(mat["mn"][0]), int(mat["kb"][0])
    byts = np.array([[int(x) for x in f[1:]] for f in sec["matrix"] if f[0] == "bytes"])
    want = np.zeros((1, (kb + 3) // 4, (mn + 3) // 4 * 4), np.uint32)
    for f in sec["matrix"]:
        if f[0] == "words":
            want[0, int(f[1])] = [int(w, 16) for w in f[2:]]
    sf = np.ldexp(np.float32(1.0), byts - 127).astype(np.float32)[None]
    words, bad = oracle.pack_sf_ue8m0(sf)
    assert bad == 0
    assert words.shape == want.shape
    assert np.array_equal(words.view(np.uint32), want)
    assert np.array_equal(oracle.unpack_sf_ue8m0(words, mn, kb)[0], byts)


def test_bf16_rne():
    rows = _rows("bf16_rne.txt")
    xs = np.array([float(Fraction(int(m)) * Fraction(2) ** int(e)) for m, e, _ in rows])
    # every value is exactly representable in float64 (at most 53 significant bits)
    for (m, e, _), x in zip(rows, xs):
        assert Fraction(x) == Fraction(int(m)) * Fraction(2) ** int(e)
    got = oracle.bf16_bits_from_f64(xs)
    want = np.array([int(b, 16) for _, _, b in rows], np.uint16)
    assert np.array_equal(got, want), [(r, hex(g)) for r, g, w in zip(rows, got, want) if g != w]


def _fill(pattern, K0):
    """One 128-wide K block of E4M3 codes from a fixture pattern."""
    kind = pattern[0]
    if kind == "alt":
        c0, c1 = int(pattern[1], 16), int(pattern[2], 16)
        return np.where(np.arange(K0) % 2 == 0, c0, c1).astype(np.uint8)
    assert kind == "fill"
    out = np.full(K0, int(pattern[1], 16), np.uint8)
    if len(pattern) > 2:
        assert pattern[2] == "at"
        out[int(pattern[3])] = int(pattern[4], 16)
    return out


def _words(exps, mn):
    """Packed scale words [1][ceil(Kb/4)][align4(mn)] written out directly:
    byte j of word [kp][r] is the biased exponent of K block 4*kp + j."""
    kb = len(exps[0])
    w = np.zeros((1, (kb + 3) // 4, (mn + 3) // 4 * 4), np.uint32)
    for r, row in enumerate(exps):
        for k, e in enumerate(row):
            w[0, k // 4, r] |= np.uint32((e + 127) << (8 * (k % 4)))
    return w.view(np.int32)


def test_gemm_worked_example():
    sec = _sections("gemm_worked_example.txt")
    shape = {f[0]: int(f[1]) for f in sec["shape"]}
    M, N, K = shape["M"], shape["N"], shape["K"]
    Kb = K // 128
    a = np.zeros((M, K), np.uint8)
    for f in sec["a"]:
        m, kb = int(f[0]), int(f[1])
        a[m, kb * 128:(kb + 1) * 128] = _fill(f[2:], 128)
    b = np.zeros((N, K), np.uint8)
    for f in sec["b"]:
        b[int(f[0])] = np.concatenate([_fill(f[1:], 128)] * Kb)
    ea = [[int(x) for x in f[1:]] for f in sorted(sec["sa"], key=lambda f: int(f[0]))]
    eb = [[int(x) for x in f[1:]] for f in sorted(sec["sb"], key=lambda f: int(f[0]))]
    sfa, sfb = _words(ea, M), _words(eb, (N + 127) // 128)

    exact = oracle.fp8_gemm_nt_f64(a, sfa, b, sfb, M, N, K)
    bits = oracle.fp8_gemm_nt(a, sfa, b, sfb, M, N, K)
    assert len(sec["d"]) == M * N
    for m, n, val, bf in sec["d"]:
        m, n = int(m), int(n)
        assert Fraction(exact[m, n]) == Fraction(val), (m, n, exact[m, n])
        assert bits[m, n] == int(bf, 16), (m, n, hex(bits[m, n]))


SENTINEL = 0xDEAD


def _grouped_inputs(sec):
    G = 1 + max(int(f[0]) for f in sec["experts"])
    b = np.zeros((G, 2, 128), np.uint8)
    for e, n, code in sec["experts"]:
        b[int(e), int(n)] = int(code, 16)
    sfb = np.concatenate([_words([[int(x)]], 1) for _, x in sorted(sec["sfb"], key=lambda f: int(f[0]))])
    return G, b, sfb


def _check_d(d, rows_expected, key_len):
    written = set()
    for f in rows_expected:
        idx = tuple(int(x) for x in f[:key_len])
        v0, v1, b0, b1 = f[key_len:]
        assert d[idx].tolist() == [int(b0, 16), int(b1, 16)], (idx, [hex(x) for x in d[idx]])
        assert Fraction(float(oracle.bf16_bits_to_f64(d[idx])[0])) == Fraction(v0)
        assert Fraction(float(oracle.bf16_bits_to_f64(d[idx])[1])) == Fraction(v1)
        written.add(idx)
    return written


def test_contiguous_worked_example():
    sec = _sections("grouped_worked_example.txt")
    G, b, sfb = _grouped_inputs(sec)
    rows = sec["contiguous"]
    M = len(rows)
    a = np.stack([np.full(128, int(code, 16), np.uint8) for _, code, _, _ in rows])
    sfa = _words([[int(x)] for _, _, x, _ in rows], M)
    m_idx = np.array([int(f[3]) for f in rows], np.int32)

    d = np.full((M, 2), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, m_idx, d, G, 2, 128) == 0
    written = _check_d(d, sec["contiguous_d"], 1)
    for m in range(M):
        if (m,) not in written:
            assert (d[m] == SENTINEL).all(), m

    kind, row, index, reported = next(f for f in sec["errors"] if f[0] == "contiguous_index")
    bad_idx = m_idx.copy()
    bad_idx[int(row)] = int(index)
    d2 = np.full((M, 2), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, bad_idx, d2, G, 2, 128) == int(reported)
    assert (d2[int(row)] == SENTINEL).all()
    others = [m for m in range(M) if m != int(row)]
    assert np.array_equal(d2[others], d[others])


def test_masked_worked_example():
    sec = _sections("grouped_worked_example.txt")
    G, b, sfb = _grouped_inputs(sec)
    M_max = 1 + max(int(f[1]) for f in sec["masked"])
    a = np.zeros((G, M_max, 128), np.uint8)
    ea = [[[0] for _ in range(M_max)] for _ in range(G)]
    for g, r, code, x in sec["masked"]:
        a[int(g), int(r)] = int(code, 16)
        ea[int(g)][int(r)] = [int(x)]
    sfa = np.concatenate([_words(ea[g], M_max) for g in range(G)])
    mm = np.array([int(x) for x in sec["masked_m"][0]], np.int32)

    d = np.full((G, M_max, 2), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, mm, d, G, M_max, 2, 128) == 0
    written = _check_d(d, sec["masked_d"], 2)
    for g in range(G):
        for r in range(M_max):
            if (g, r) not in written:
                assert (d[g, r] == SENTINEL).all(), (g, r)

    kind, g, count, reported = next(f for f in sec["errors"] if f[0] == "masked_count")
    mm2 = mm.copy()
    mm2[int(g)] = int(count)
    d2 = np.full((G, M_max, 2), SENTINEL, np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, mm2, d2, G, M_max, 2, 128) == int(reported)
    assert np.array_equal(d2, d)
