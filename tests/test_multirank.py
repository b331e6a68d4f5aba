"""Multi-process (gloo, world size 2, CPU) tests of the host logic used when
the GEMMs run on several GPUs: sharding into independent problems and the
max-over-ranks timing reduction.  Each rank computes its shard with the CPU
oracle; gathering the shards must reproduce the unsharded result exactly."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from moe_grouped_gemm_05_b200 import shard, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, fn, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q.put((rank, fn(rank, world)))
    except Exception as e:  # noqa: BLE001 - report to the parent
        q.put((rank, e))
    finally:
        dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fn, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, v = q.get(timeout=120)
        out[r] = v
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, v in out.items():
        if isinstance(v, Exception):
            raise v
    return [out[r] for r in range(world)]


def _rank_masked(rank, world):
    p = synth.masked_problem(5, 128, 256, 256, seed=51, masked_m=[100, 0, 128, 7, 60])
    owned = shard.partition_experts(p.masked_m, world)[rank]
    sa, _ = oracle.pack_sf_ue8m0(p.sfa)
    sb, _ = oracle.pack_sf_ue8m0(p.sfb)
    d = np.zeros((p.G, p.M, p.N), np.uint16)
    for g in owned:
        mg = int(p.masked_m[g])
        if mg:
            d[g, :mg] = oracle.fp8_gemm_nt(p.a[g], sa[g], p.b[g], sb[g], p.M, p.N, p.K, rows=np.arange(mg))
    gathered = [None] * world
    dist.all_gather_object(gathered, (owned, d))
    t = shard.max_over_ranks(1.0 + rank)
    return gathered, t


def _rank_dense(rank, world):
    p = synth.dense_problem(64, 640, 256, seed=52)
    n0, n1 = shard.split_n(p.N, world, rank)
    sa, _ = oracle.pack_sf_ue8m0(p.sfa[None])
    # this rank's B rows and its contiguous slice of B's 128-row scale blocks
    sb, _ = oracle.pack_sf_ue8m0(p.sfb[None, n0 // 128:(n1 + 127) // 128])
    d = oracle.fp8_gemm_nt(p.a, sa[0], p.b[n0:n1], sb[0], p.M, n1 - n0, p.K)
    gathered = [None] * world
    dist.all_gather_object(gathered, (n0, n1, d))
    return gathered


def _rank_contiguous(rank, world):
    counts = [300, 0, 40, 128, 77]
    p = synth.contiguous_problem(5, 256, 256, rows=0, seed=53, counts=counts)
    owned = shard.partition_experts(counts, world)[rank]
    src, loc = shard.local_contiguous_layout(p.m_indices, owned)
    take = np.maximum(src, 0)
    a = p.a[take]                                   # padding rows: any bytes, never read into D
    sa, _ = oracle.pack_sf_ue8m0(p.sfa[take][None])
    sb, _ = oracle.pack_sf_ue8m0(p.sfb[owned]) if owned else (np.zeros((0, 1, 4), np.int32), 0)
    d_local = np.zeros((len(src), p.N), np.uint16)
    if owned:
        assert oracle.m_grouped_fp8_gemm_nt_contiguous(a, sa[0], p.b[owned], sb, loc, d_local, len(owned),
                                                       p.N, p.K) == 0
    d = np.zeros((p.M, p.N), np.uint16)
    d[src[src >= 0]] = d_local[src >= 0]
    gathered = [None] * world
    dist.all_gather_object(gathered, (owned, d, len(src) % 128))
    return gathered


@pytest.mark.timeout(300)
def test_expert_parallel_contiguous_equals_unsharded():
    gathered = _run(_rank_contiguous)[0]
    p = synth.contiguous_problem(5, 256, 256, rows=0, seed=53, counts=[300, 0, 40, 128, 77])
    sa, _ = oracle.pack_sf_ue8m0(p.sfa[None])
    sb, _ = oracle.pack_sf_ue8m0(p.sfb)
    ref = np.zeros((p.M, p.N), np.uint16)
    assert oracle.m_grouped_fp8_gemm_nt_contiguous(p.a, sa[0], p.b, sb, p.m_indices, ref, p.G, p.N, p.K) == 0
    assert sorted(g for owned, _, _ in gathered for g in owned) == list(range(p.G))
    merged = np.zeros_like(ref)
    for owned, d, tail in gathered:
        assert tail == 0                              # local segments stay 128-aligned
        rows = np.isin(p.m_indices, owned)
        merged[rows] = d[rows]
        assert (d[~rows] == 0).all()                  # a rank writes only its experts' rows
    assert np.array_equal(merged, ref)


def test_local_contiguous_layout_by_hand():
    m_idx = np.array([0, 0, -1, -1, 2, -1, 1, 1, 1, -1], np.int32)
    src, loc = shard.local_contiguous_layout(m_idx, [1, 2], align=4)
    assert src.tolist() == [6, 7, 8, -1, 4, -1, -1, -1]
    assert loc.tolist() == [0, 0, 0, -1, 1, -1, -1, -1]
    src, loc = shard.local_contiguous_layout(m_idx, [], align=4)
    assert len(src) == 0 and len(loc) == 0


@pytest.mark.timeout(300)
def test_expert_parallel_masked_equals_unsharded():
    results = _run(_rank_masked)
    p = synth.masked_problem(5, 128, 256, 256, seed=51, masked_m=[100, 0, 128, 7, 60])
    sa, _ = oracle.pack_sf_ue8m0(p.sfa)
    sb, _ = oracle.pack_sf_ue8m0(p.sfb)
    ref = np.zeros((p.G, p.M, p.N), np.uint16)
    oracle.m_grouped_fp8_gemm_nt_masked(p.a, sa, p.b, sb, p.masked_m, ref, p.G, p.M, p.N, p.K)
    gathered, t0 = results[0]
    assert t0 == 2.0 and results[1][1] == 2.0          # max over ranks
    owned = [o for o, _ in gathered]
    assert sorted(g for o in owned for g in o) == list(range(p.G))  # each expert exactly once
    full = np.zeros_like(ref)
    for o, d in gathered:
        for g in o:
            full[g] = d[g]
    assert np.array_equal(full, ref)


@pytest.mark.timeout(300)
def test_n_sharded_dense_equals_unsharded():
    gathered = _run(_rank_dense)[0]
    p = synth.dense_problem(64, 640, 256, seed=52)
    sa, _ = oracle.pack_sf_ue8m0(p.sfa[None])
    sb, _ = oracle.pack_sf_ue8m0(p.sfb[None])
    ref = oracle.fp8_gemm_nt(p.a, sa[0], p.b, sb[0], p.M, p.N, p.K)
    cols = sorted((n0, n1) for n0, n1, _ in gathered)
    assert cols[0][0] == 0 and cols[-1][1] == p.N and cols[0][1] == cols[1][0]
    full = np.concatenate([d for _, _, d in sorted(gathered, key=lambda x: x[0])], axis=1)
    assert np.array_equal(full, ref)


def test_partition_experts_balances_rows():
    rows = synth.zipf_counts(7, 32768, 8, 1.1)
    parts = shard.partition_experts(rows, 4)
    assert sorted(g for p in parts for g in p) == list(range(8))
    loads = [int(rows[p].sum()) for p in parts]
    assert max(loads) - min(loads) <= int(rows.max())  # LPT bound
    assert shard.partition_experts([5, 5, 5], 2) == shard.partition_experts([5, 5, 5], 2)


def test_split_n_covers_whole_blocks():
    for N in (640, 7168, 4096 + 16):
        for world in (1, 2, 3, 8):
            ranges = [shard.split_n(N, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == N
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0 and a0 % 128 == 0
    with pytest.raises(ValueError):
        shard.split_n(128, 2, 2)
