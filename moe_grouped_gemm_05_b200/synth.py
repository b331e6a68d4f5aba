"""Seeded synthetic inputs for the FP8 block-scaled GEMMs.

This module is shared by the tests, the benchmark and the CPU oracle's
tests.  It only *draws* inputs: a counter-based SplitMix64 stream, the
Box-Muller transform, Zipf/uniform routing draws and the test-input
quantisation recipe (per-1x128 / per-128x128 amax scaled to a power of two,
cast to E4M3 with PyTorch's own ``float8_e4m3fn`` conversion).  It holds none
of the GEMM's arithmetic: no E4M3/UE8M0 decoding, no scale packing, no
products, sums or output rounding.

Workloads (DeepGEMM pages: "DeepGEMM 简介" / "三种 GEMM 类型支持" — dense NT,
contiguous M-grouped, masked M-grouped):

* values are N(0, sigma) fp32 drawn from SplitMix64 + Box-Muller;
* A gets one power-of-two scale per row and 128-wide K group, B one per
  128x128 block; scale = 2**ceil(log2(amax/448)), 1.0 for an all-zero group;
* contiguous routing: rows drawn i.i.d. from a Zipf(s) categorical over the
  experts, each expert segment padded with index -1 to a multiple of 128;
* masked routing: valid rows per expert drawn uniformly from {0..M_max}.
"""
from __future__ import annotations

import dataclasses
import math
import os

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
E4M3_MAX = 448.0
BLOCK = 128


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the SplitMix64 stream for ``seed``.

    Output i is mix(seed + (i+1) * golden) with the published SplitMix64
    finaliser, so any slice of the stream can be drawn independently.
    """
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, start: int, count: int) -> np.ndarray:
    """Uniform doubles in [0, 1) from the top 53 bits of SplitMix64."""
    z = splitmix64(seed, start, count)
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, count: int, sigma: float = 1.0, chunk: int = 1 << 21) -> np.ndarray:
    """``count`` N(0, sigma) fp32 values (Box-Muller over consecutive pairs).

    Pair i uses stream outputs 2i and 2i+1 only, so chunks of pairs are drawn
    independently (on a thread pool: NumPy's ufuncs release the GIL) and the
    result does not depend on the chunking."""
    out = np.empty(count, dtype=np.float32)
    pairs = (count + 1) // 2

    def fill(done: int) -> None:
        n = min(chunk, pairs - done)
        u = uniform01(seed, 2 * done, 2 * n)
        u1 = 1.0 - u[0::2]  # (0, 1]
        u2 = u[1::2]
        r = np.sqrt(-2.0 * np.log(u1)) * sigma
        t = 2.0 * math.pi * u2
        z = np.empty(2 * n, dtype=np.float64)
        z[0::2] = r * np.cos(t)
        z[1::2] = r * np.sin(t)
        lo = 2 * done
        hi = min(count, lo + 2 * n)
        out[lo:hi] = z[: hi - lo].astype(np.float32)

    starts = range(0, pairs, chunk)
    if pairs <= chunk:
        for s in starts:
            fill(s)
    else:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    return out


def _pow2_scale(amax: np.ndarray) -> np.ndarray:
    """Smallest power of two s with amax / s <= 448 (1.0 where amax == 0)."""
    r = amax.astype(np.float64) / E4M3_MAX
    f, e = np.frexp(r)
    c = np.where(f == 0.5, e - 1, e)
    s = np.ldexp(1.0, c)
    return np.where(amax > 0, s, 1.0).astype(np.float32)


def _to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def quantize_rows(x: np.ndarray):
    """Per-row, per-128-column quantisation of ``x[..., R, K]`` (the A recipe).

    Returns (E4M3 bytes with x's shape, fp32 power-of-two scales [..., R, K/128]).
    """
    *lead, R, K = x.shape
    assert K % BLOCK == 0
    g = x.reshape(*lead, R, K // BLOCK, BLOCK)
    s = _pow2_scale(np.abs(g).max(axis=-1))
    q = _to_e4m3_bytes(g / s[..., None]).reshape(x.shape)
    return q, s


def quantize_blocks(x: np.ndarray):
    """Per-128x128-block quantisation of ``x[..., R, K]`` (the B recipe).

    Returns (E4M3 bytes with x's shape, fp32 scales [..., ceil(R/128), K/128]).
    """
    *lead, R, K = x.shape
    assert K % BLOCK == 0
    rb = (R + BLOCK - 1) // BLOCK
    pad = rb * BLOCK - R
    xp = x if pad == 0 else np.concatenate([x, np.zeros((*lead, pad, K), np.float32)], axis=-2)
    g = xp.reshape(*lead, rb, BLOCK, K // BLOCK, BLOCK)
    s = _pow2_scale(np.abs(g).max(axis=(-3, -1)))
    q = _to_e4m3_bytes(g / s[..., None, :, None]).reshape(xp.shape)
    if pad:
        q = q[..., :R, :]
    return np.ascontiguousarray(q), s


def zipf_counts(seed: int, rows: int, groups: int, s: float) -> np.ndarray:
    """Rows per expert when ``rows`` tokens are drawn i.i.d. from Zipf(s) over ranks 1..groups."""
    p = np.arange(1, groups + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(p / p.sum())
    cdf[-1] = 1.0
    u = uniform01(seed, 0, rows)
    e = np.searchsorted(cdf, u, side="right")
    return np.bincount(e, minlength=groups).astype(np.int64)


def topk_routing(seed: int, tokens: int, topk: int, groups: int, s: float = 1.1):
    """Top-k routing of ``tokens`` tokens over ``groups`` experts: each token's
    ``topk`` distinct experts drawn without replacement with Zipf(s) weights
    over ranks 1..groups (the largest of log w_e + Gumbel noise, the noise
    from SplitMix64 uniforms), and gate weights that sum to one per token.
    Returns (ids int32 [tokens, topk], gates float32 [tokens, topk])."""
    w = np.arange(1, groups + 1, dtype=np.float64) ** (-s)
    u = np.clip(uniform01(seed, 0, tokens * groups), 1e-300, None).reshape(tokens, groups)
    keys = np.log(w)[None, :] - np.log(-np.log(u))
    ids = np.argsort(-keys, axis=1, kind="stable")[:, :topk].astype(np.int32)
    g = uniform01(seed ^ 0x5151, 0, tokens * topk).reshape(tokens, topk) + 0.5
    return ids, (g / g.sum(axis=1, keepdims=True)).astype(np.float32)


def contiguous_indices(counts: np.ndarray, align: int = BLOCK) -> np.ndarray:
    """Per-row expert index for segments of ``counts`` rows, each padded with -1 to ``align``."""
    parts = []
    for g, c in enumerate(counts):
        padded = -(-int(c) // align) * align
        seg = np.full(padded, -1, dtype=np.int32)
        seg[: int(c)] = g
        parts.append(seg)
    return np.concatenate(parts) if parts else np.zeros(0, np.int32)


def uniform_masked_m(seed: int, groups: int, m_max: int) -> np.ndarray:
    """Valid rows per expert, each uniform on {0, ..., m_max}."""
    u = uniform01(seed, 0, groups)
    return np.minimum(np.floor(u * (m_max + 1)), m_max).astype(np.int32)


def choose_rows(seed: int, total: int, k: int) -> np.ndarray:
    """``k`` distinct row indices out of ``total`` (partial Fisher-Yates on SplitMix64)."""
    perm = np.arange(total)
    u = uniform01(seed, 0, k)
    for i in range(k):
        j = i + int(u[i] * (total - i))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:k])


# --------------------------------------------------------------------------
# Named workloads


@dataclasses.dataclass
class Problem:
    """One synthetic problem: E4M3 operands, fp32 power-of-two scales, routing."""

    kind: str            # "dense" | "contiguous" | "masked"
    name: str
    a: np.ndarray        # uint8 E4M3: [M,K] | [M_total,K] | [G,M_max,K]
    sfa: np.ndarray      # fp32: [M,Kb] | [M_total,Kb] | [G,M_max,Kb]
    b: np.ndarray        # uint8 E4M3: [N,K] | [G,N,K]
    sfb: np.ndarray      # fp32: [ceil(N/128),Kb] | [G,ceil(N/128),Kb]
    M: int               # rows (dense), total rows (contiguous), M_max (masked)
    N: int
    K: int
    G: int = 1
    m_indices: np.ndarray | None = None
    masked_m: np.ndarray | None = None

    @property
    def valid_rows(self) -> int:
        if self.kind == "dense":
            return self.M
        if self.kind == "contiguous":
            return int((self.m_indices >= 0).sum())
        return int(self.masked_m.sum())

    @property
    def flops(self) -> float:
        """Algorithmic work, 2*M*N*K with M the valid rows only (discosf.com
        DeepGEMM tutorial, section 4.3: one multiply and one add per term;
        padding and masked-out rows do no useful work and are not counted)."""
        return 2.0 * self.valid_rows * self.N * self.K


def dense_problem(M, N, K, seed, sigma_a=1.0, sigma_b=1.0, outlier_frac=0.0, outlier_mul=64.0,
                  name=None) -> Problem:
    a = normal(seed, M * K, sigma_a).reshape(M, K)
    if outlier_frac > 0:
        rows = choose_rows(seed ^ 0x5A5A, M, int(round(outlier_frac * M)))
        a[rows] *= np.float32(outlier_mul)
    b = normal(seed + 0x10000, N * K, sigma_b).reshape(N, K)
    qa, sa = quantize_rows(a)
    qb, sb = quantize_blocks(b)
    return Problem("dense", name or f"dense_{M}x{N}x{K}", qa, sa, qb, sb, M, N, K)


def contiguous_problem(G, N, K, rows, seed, zipf_s=1.1, counts=None, name=None) -> Problem:
    if counts is None:
        counts = zipf_counts(seed ^ 0x2121, rows, G, zipf_s)
    m_idx = contiguous_indices(np.asarray(counts))
    Mt = len(m_idx)
    a = normal(seed, Mt * K).reshape(Mt, K)
    b = normal(seed + 0x10000, G * N * K).reshape(G, N, K)
    qa, sa = quantize_rows(a)
    qb, sb = quantize_blocks(b)
    return Problem("contiguous", name or f"contiguous_{G}x{N}x{K}", qa, sa, qb, sb, Mt, N, K, G,
                   m_indices=m_idx)


def masked_problem(G, M_max, N, K, seed, masked_m=None, name=None) -> Problem:
    if masked_m is None:
        masked_m = uniform_masked_m(seed ^ 0x3131, G, M_max)
    a = normal(seed, G * M_max * K).reshape(G, M_max, K)
    b = normal(seed + 0x10000, G * N * K).reshape(G, N, K)
    qa, sa = quantize_rows(a)
    qb, sb = quantize_blocks(b)
    return Problem("masked", name or f"masked_{G}x{M_max}x{N}x{K}", qa, sa, qb, sb, M_max, N, K, G,
                   masked_m=np.asarray(masked_m, dtype=np.int32))


WORKLOADS = {
    # small dense case the oracle finishes in well under a second
    "dense_128x512x512": lambda: dense_problem(128, 512, 512, 1000),
    # the headline dense shape (tensor-core bound)
    "dense_4096x7168x2048": lambda: dense_problem(4096, 7168, 2048, 1001),
    # dense decode shape (HBM bound)
    "dense_64x7168x2048": lambda: dense_problem(64, 7168, 2048, 1001 + 0x100),
    # 8 experts, N=4096, K=7168, 32768 Zipf(1.1)-routed rows
    "contiguous_8x4096x7168_zipf1.1": lambda: contiguous_problem(8, 4096, 7168, 32768, 1002),
    # 16 experts, up to 256 rows each, N=7168, K=2048
    "masked_16x256x7168x2048": lambda: masked_problem(16, 256, 7168, 2048, 1003),
    # 8192^3 with 1% outlier rows (x64) in A and B ~ N(0, 0.02)
    "dense_8192x8192x8192_outliers": lambda: dense_problem(8192, 8192, 8192, 1004, sigma_b=0.02,
                                                           outlier_frac=0.01),
}
