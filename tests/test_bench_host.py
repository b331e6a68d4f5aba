"""Host-side bookkeeping of the benchmark: the algorithmic bytes behind the
roofline fraction, the choice of bound, and the rule that recorded DRAM
traffic is reported only for the kernel code and configuration it was taken on."""
import json
import os
import sys
from types import SimpleNamespace

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _dense(M, N, K):
    return SimpleNamespace(kind="dense", M=M, N=N, K=K, G=1, valid_rows=M, flops=2.0 * M * N * K)


def test_dense_bytes_by_hand():
    # 4096 x 7168 x 2048: A 4096*2048, B 7168*2048, D 2*4096*7168, scales (4096 + 56) * 16 bytes
    assert bench.algorithmic_bytes(_dense(4096, 7168, 2048)) == 8388608 + 14680064 + 58720256 + 66432
    # 64-row decode: A 64*2048, B 7168*2048, D 2*64*7168, scales (64 + 56) * 16
    assert bench.algorithmic_bytes(_dense(64, 7168, 2048)) == 131072 + 14680064 + 917504 + 1920


def test_grouped_bytes_count_only_valid_rows_and_used_experts():
    N, K = 256, 512                      # 2 N blocks, 4 K blocks
    m_idx = np.array([0] * 100 + [-1] * 28 + [2] * 128, np.int32)   # expert 1 has no rows
    p = SimpleNamespace(kind="contiguous", M=256, N=N, K=K, G=3, valid_rows=228, m_indices=m_idx,
                        flops=2.0 * 228 * N * K)
    per_expert = N * K + 2 * 4
    assert bench.algorithmic_bytes(p) == 228 * (K + 4) + 2 * per_expert + 2 * 228 * N
    mm = np.array([3, 0, 0, 5], np.int32)
    q = SimpleNamespace(kind="masked", M=8, N=N, K=K, G=4, valid_rows=8, masked_m=mm, flops=2.0 * 8 * N * K)
    assert bench.algorithmic_bytes(q) == 8 * (K + 4) + 2 * per_expert + 2 * 8 * N


@pytest.mark.parametrize("shape,bound", [((4096, 7168, 2048), "tensor"), ((8192, 8192, 8192), "tensor"),
                                         ((64, 7168, 2048), "hbm")])
def test_bound_of_dense_shapes(shape, bound):
    assert bench.bound_of(_dense(*shape)) == bound


def test_bound_of_masked_decode_is_hbm():
    mm = np.full(16, 82, np.int32)       # ~1310 rows over 16 experts
    p = SimpleNamespace(kind="masked", M=256, N=7168, K=2048, G=16, valid_rows=int(mm.sum()), masked_m=mm,
                        flops=2.0 * int(mm.sum()) * 7168 * 2048)
    assert bench.bound_of(p) == "hbm"


def test_recorded_traffic_requires_same_code_and_configuration(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    rec = {"w": {"kernel_hash": "abc", "kernel_config": "256x224", "dram_bytes_per_launch": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.recorded_traffic("w", "256x224") == 123
    assert bench.recorded_traffic("w", "128x224") is None      # another configuration
    assert bench.recorded_traffic("other", "256x224") is None  # another workload
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "def")
    assert bench.recorded_traffic("w", "256x224") is None      # the kernel changed since


def test_committed_traffic_records_are_consistent():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert rec
    for e in rec.values():
        assert e["dram_bytes_per_launch"] == e["dram_read_bytes"] + e["dram_write_bytes"]
        assert e["kernel_hash"] and e["kernel_config"] and os.path.exists(os.path.join(ROOT, e["source"].split()[0]))


def _contig_problem():
    from moe_grouped_gemm_05_b200 import synth

    return synth.contiguous_problem(5, 384, 256, rows=700, seed=11)


def test_shard_problem_n_split_covers_every_column_once():
    from moe_grouped_gemm_05_b200 import synth

    p = synth.dense_problem(64, 1408, 256, seed=3)
    parts = [bench.shard_problem(p, 3, r, "n") for r in range(3)]
    assert sum(q.N for q in parts) == p.N and all(q.N % 128 == 0 for q in parts)
    assert np.array_equal(np.concatenate([q.b for q in parts]), p.b)
    assert np.array_equal(np.concatenate([q.sfb for q in parts]), p.sfb)
    assert sum(q.flops for q in parts) == p.flops
    assert bench.shard_problem(p, 1, 0, "n") is p


def test_shard_problem_experts_keeps_every_valid_row_once():
    p = _contig_problem()
    seen = []
    for r in range(2):
        q = bench.shard_problem(p, 2, r, "experts")
        assert q.M % 128 == 0 and q.a.shape == (q.M, p.K) and q.b.shape[0] == q.G
        valid = q.m_indices >= 0
        # every local row holds one of the global rows of an owned expert, with its codes and scales
        for i in np.nonzero(valid)[0][:50]:
            j = np.nonzero((p.a == q.a[i]).all(axis=1))[0]
            assert len(j) >= 1 and p.m_indices[j[0]] >= 0
        seen.append(int(valid.sum()))
    assert sum(seen) == p.valid_rows


def test_weak_scaling_job_problem():
    """Weak scaling: P ranks each own a headline-sized share of a problem P
    times larger (along N, or in experts and their routed rows); the job's
    FLOP are P times the headline's, and one rank is the headline itself."""
    from moe_grouped_gemm_05_b200 import synth

    p = _contig_problem()
    one = bench.global_problem(p, 1, "n")
    assert (one["N"], one["G"], one["M"], one["flops"]) == (p.N, p.G, p.M, p.flops)
    g = bench.global_problem(p, 4, "n")
    assert (g["N"], g["G"], g["M"]) == (4 * p.N, p.G, p.M) and g["flops"] == 4 * p.flops
    # N-split shares of the job problem are each the headline's N columns
    assert g["N"] // 4 == p.N
    e = bench.global_problem(p, 4, "experts")
    assert (e["N"], e["G"], e["M"], e["valid_rows"]) == (p.N, 4 * p.G, 4 * p.M, 4 * p.valid_rows)
    assert e["flops"] == 4 * p.flops
    d = synth.dense_problem(64, 256, 256, seed=4)
    assert bench.global_problem(d, 2, "experts")["N"] == 2 * d.N  # dense problems always split N
    m = synth.masked_problem(3, 128, 256, 256, seed=5)
    mg = bench.global_problem(m, 2, "experts")
    assert (mg["G"], mg["M"], mg["valid_rows"]) == (6, m.M, 2 * m.valid_rows)
