"""Host-side partitioning of the GEMMs across GPUs (one process per GPU).

The FP8 GEMMs have no exchange step: K is never split, so every output
element is computed on one GPU.  A multi-GPU job therefore shards into
independent problems and needs no collective on the data path:

* dense GEMM: each rank takes a range of N (whole 128-column scale blocks,
  so each rank's B scales are a contiguous slice of the packed words) or
  simply runs its own independent problem (weak scaling);
* grouped GEMMs: expert parallelism -- each rank owns a set of experts.
  :func:`partition_experts` balances the ranks by valid rows (the cost of an
  expert is proportional to its rows, [DeepGEMM pages: M-axis-only grouping,
  N and K shared by all experts]).

The only collectives a job needs are for timing and bookkeeping
(:func:`max_over_ranks`).
"""
from __future__ import annotations

import heapq

import numpy as np


def split_n(N: int, world: int, rank: int, align: int = 128) -> tuple[int, int]:
    """Column range [n0, n1) of rank `rank` when N is split into `world` parts of whole `align` blocks."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    blocks = -(-N // align)
    lo = rank * blocks // world
    hi = (rank + 1) * blocks // world
    return min(N, lo * align), min(N, hi * align)


def partition_experts(rows_per_expert, world: int) -> list[list[int]]:
    """Assigns experts to `world` ranks, largest first to the least-loaded rank.

    Returns, per rank, the sorted list of expert ids.  Every expert appears
    exactly once; ties go to the lower rank, so the result is deterministic.
    """
    rows = np.asarray(rows_per_expert, dtype=np.int64)
    if world <= 0:
        raise ValueError("world must be positive")
    order = sorted(range(len(rows)), key=lambda g: (-int(rows[g]), g))
    heap = [(0, r) for r in range(world)]
    heapq.heapify(heap)
    owned: list[list[int]] = [[] for _ in range(world)]
    for g in order:
        load, r = heapq.heappop(heap)
        owned[r].append(g)
        heapq.heappush(heap, (load + int(rows[g]), r))
    return [sorted(o) for o in owned]


def local_contiguous_layout(m_indices, owned, align: int = 128):
    """This rank's contiguous layout when it owns the experts in ``owned``.

    The owned experts' rows are taken from the global contiguous layout in
    expert order (the order of ``owned``), keeping their order within each
    expert, and each expert's segment is padded with -1 to a multiple of
    ``align`` rows.  Returns ``(src_rows, local_m_indices)``, both int32 of
    the local row count: ``src_rows[i]`` is the global row that local row ``i``
    holds (-1 for padding), and ``local_m_indices[i]`` its expert's position
    in ``owned`` (-1 for padding).  Scattering the local output rows back to
    ``src_rows`` reproduces the global output of those experts.
    """
    m_indices = np.asarray(m_indices)
    src, loc = [], []
    for j, g in enumerate(owned):
        rows = np.nonzero(m_indices == g)[0]
        padded = -(-len(rows) // align) * align
        seg_src = np.full(padded, -1, np.int32)
        seg_src[:len(rows)] = rows
        seg_loc = np.full(padded, -1, np.int32)
        seg_loc[:len(rows)] = j
        src.append(seg_src)
        loc.append(seg_loc)
    if not src:
        return np.zeros(0, np.int32), np.zeros(0, np.int32)
    return np.concatenate(src), np.concatenate(loc)


def max_over_ranks(value: float, group=None) -> float:
    """Maximum of `value` over all ranks of the default process group (identity when not distributed)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
