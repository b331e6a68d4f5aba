"""Shared test helpers: moving synthetic problems to the GPU, the oracle's
packed scales, and the parity tolerance.

Tolerance for BF16 outputs (per valid row m, per column n):
    |gpu - ref| <= ulp_bf16(ref) + 2^-10 * max_n |ref[m, n]|
and, over all valid rows of one call, the normalised difference
    1 - 2 sum(x*y) / sum(x^2 + y^2) < 1e-4.
Integer-valued problems must match bit for bit.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from moe_grouped_gemm_05_b200 import synth


def packed(problem: synth.Problem):
    """Oracle-packed scale words (int32 numpy) for A and B of a problem."""
    if problem.kind == "masked":
        sa, bad_a = oracle.pack_sf_ue8m0(problem.sfa)
    else:
        sa, bad_a = oracle.pack_sf_ue8m0(problem.sfa[None])
        sa = sa[0]
    if problem.kind == "dense":
        sb, bad_b = oracle.pack_sf_ue8m0(problem.sfb[None])
        sb = sb[0]
    else:
        sb, bad_b = oracle.pack_sf_ue8m0(problem.sfb)
    assert bad_a == 0 and bad_b == 0
    return sa, sb


def to_device(problem: synth.Problem, sa=None, sb=None, dev="cuda"):
    if sa is None:
        sa, sb = packed(problem)
    t = {
        "a": torch.from_numpy(problem.a).to(dev).view(torch.float8_e4m3fn),
        "b": torch.from_numpy(problem.b).to(dev).view(torch.float8_e4m3fn),
        "sfa": torch.from_numpy(np.ascontiguousarray(sa)).to(dev),
        "sfb": torch.from_numpy(np.ascontiguousarray(sb)).to(dev),
    }
    if problem.m_indices is not None:
        t["m_indices"] = torch.from_numpy(problem.m_indices).to(dev)
    if problem.masked_m is not None:
        t["masked_m"] = torch.from_numpy(problem.masked_m).to(dev)
    return t


def bits(d: torch.Tensor) -> np.ndarray:
    return d.view(torch.int16).cpu().numpy().view(np.uint16)


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    _, e = np.frexp(np.where(ax > 0, ax, 1.0))
    lg = e - 1
    return np.where(ax >= 2.0 ** -126, np.ldexp(1.0, lg - 7), 2.0 ** -133)


def check_close(got_bits: np.ndarray, ref_bits: np.ndarray, what: str = ""):
    """Asserts the BF16 tolerance on 2-D arrays of valid rows [rows, N]."""
    assert got_bits.shape == ref_bits.shape, (got_bits.shape, ref_bits.shape)
    if got_bits.size == 0:
        return
    x = oracle.bf16_bits_to_f64(got_bits)
    y = oracle.bf16_bits_to_f64(ref_bits)
    assert np.isfinite(x).all(), f"{what}: non-finite output"
    rowmax = np.abs(y).max(axis=1, keepdims=True)
    bound = ulp_bf16(y) + 2.0 ** -10 * rowmax
    err = np.abs(x - y)
    bad = err > bound
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; first at ({i},{j}): "
                             f"got {x[i, j]!r} ref {y[i, j]!r} bound {bound[i, j]!r}")
    den = float((x * x + y * y).sum())
    diff = 0.0 if den == 0 else 1.0 - 2.0 * float((x * y).sum()) / den
    assert diff < 1e-4, f"{what}: normalised difference {diff}"


def oracle_rows(a, sfa_words, b, sfb_words, M, N, K, rows, chunk: int = 256) -> np.ndarray:
    """The oracle's BF16 bits of the given output rows of D = A . B^T, computed
    in chunks of rows on a thread pool with single-threaded BLAS (each chunk
    is an independent call of the oracle, so the result is the same as one
    call over all rows)."""
    from threadpoolctl import threadpool_limits

    rows = np.asarray(rows)
    if len(rows) <= chunk:
        return oracle.fp8_gemm_nt(a, sfa_words, b, sfb_words, M, N, K, rows=rows)
    parts = [rows[i:i + chunk] for i in range(0, len(rows), chunk)]
    with threadpool_limits(1):
        with ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1))) as ex:
            out = list(ex.map(lambda r: oracle.fp8_gemm_nt(a, sfa_words, b, sfb_words, M, N, K, rows=r), parts))
    return np.concatenate(out)
