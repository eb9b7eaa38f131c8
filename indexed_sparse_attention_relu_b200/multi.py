"""Host logic for running the hot path on several GPUs of one node.

Decode sequences are independent: every rank runs the whole path on its own
sequences and no data crosses GPUs. What remains on the host is

  * assigning sequences to ranks (longest first onto the least-loaded rank,
    so ragged context lengths do not leave one GPU with the long tail: the
    load skew of "later position, longer history" that the pages describe
    for causal work applies to ragged decode batches as well), and
  * timing: every rank times its own steps with CUDA events, and the job's
    time is the maximum over ranks (a job is done when its slowest rank is).

Prefill of one long causal sequence is split by query rows instead
(context parallelism). Row t attends over history 0..t, so a contiguous
split would leave the last rank with almost all the work; the zigzag layout
of the long-sequence partitioning sections of "Optimizing Inference for New
Model Architectures ..." (section 5) and "Inference Adaptation and
Performance Optimization ..." (section 5.2) cuts the rows into 2N segments
and gives rank d segments d and 2N-1-d, pairing an early (cheap) segment
with a late (expensive) one. Each rank then needs every cache row up to its
last position: one all-gather of the index-key and KV rows the ranks
produced (each rank holds the rows of its own segments), after which every
rank runs the whole path on its own query rows, and the outputs are put
back in the original order by the inverse permutation.

All of it is plain functions of their inputs plus collectives, so it runs
under any torch.distributed backend (nccl on the GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import heapq
from typing import List, Sequence, Tuple

import numpy as np


def shard_sequences(work: Sequence[int], world: int) -> List[List[int]]:
    """Assigns sequence indices to `world` ranks, balancing the total work.

    work[b] is the cost of sequence b (its context length for decode: the
    indexer reads every cached key). Greedy longest-processing-time: the
    sequences in descending order of work, each to the rank with the least
    work so far (ties to the lower rank). Returns, per rank, its sequence
    indices in ascending order. Every index appears exactly once."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(work)), key=lambda b: (-int(work[b]), b))
    heap = [(0, r) for r in range(world)]
    heapq.heapify(heap)
    out: List[List[int]] = [[] for _ in range(world)]
    for b in order:
        load, r = heapq.heappop(heap)
        out[r].append(b)
        heapq.heappush(heap, (load + int(work[b]), r))
    return [sorted(s) for s in out]


def shard_loads(work: Sequence[int], shards: List[List[int]]) -> np.ndarray:
    """Total work per rank of an assignment."""
    return np.array([sum(int(work[b]) for b in s) for s in shards], dtype=np.int64)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The maximum of a per-rank scalar over all ranks (identity without a
    process group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: Sequence[int], max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed divided by the
    job's time (the slowest rank's), in units per second."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return float(sum(int(u) for u in units_per_rank)) / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- zigzag context parallelism

def zigzag_segments(n_rows: int, world: int) -> List[List[Tuple[int, int]]]:
    """The rows [0, n_rows) cut into 2 * world contiguous segments (sizes
    differ by at most one row), rank d getting segments d and 2*world-1-d,
    as a list of [start, end) pairs per rank, in segment order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    n_seg = 2 * world
    bounds = [n_rows * i // n_seg for i in range(n_seg + 1)]
    seg = [(bounds[i], bounds[i + 1]) for i in range(n_seg)]
    return [[seg[d], seg[n_seg - 1 - d]] for d in range(world)]


def zigzag_rows(n_rows: int, world: int, rank: int) -> np.ndarray:
    """The query rows rank `rank` processes, in ascending order."""
    return np.concatenate([np.arange(a, b, dtype=np.int64) for a, b in zigzag_segments(n_rows, world)[rank]])


def zigzag_restore(parts: Sequence[np.ndarray], n_rows: int, world: int) -> np.ndarray:
    """Inverse of the zigzag split: `parts[d]` holds rank d's results in the
    order of zigzag_rows(n_rows, world, d) (first axis); returns them in the
    original row order."""
    first = np.asarray(parts[0])
    out = np.empty((n_rows,) + first.shape[1:], dtype=first.dtype)
    for d in range(world):
        rows = zigzag_rows(n_rows, world, d)
        part = np.asarray(parts[d])
        if part.shape[0] != len(rows):
            raise ValueError(f"rank {d}: {part.shape[0]} results for {len(rows)} rows")
        out[rows] = part
    return out


def causal_work(rows: np.ndarray, history_from: int = 0) -> int:
    """Causal scoring work of query rows at positions `history_from + row`:
    each scores every position up to its own (sum of position + 1)."""
    r = np.asarray(rows, dtype=np.int64) + history_from
    return int((r + 1).sum())


def all_gather_rows(local: "torch.Tensor", dist) -> List["torch.Tensor"]:
    """Every rank's `local` rows (same trailing shape; any row count), gathered
    on every rank in rank order (sizes exchanged first, rows padded to the
    largest count for the collective and cut back)."""
    import torch

    world = dist.get_world_size()
    n = torch.tensor([local.shape[0]], dtype=torch.int64, device=local.device)
    sizes = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(sizes, n)
    sizes = [int(x.item()) for x in sizes]
    width = max(sizes)
    padded = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    padded[:local.shape[0]] = local
    bufs = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(bufs, padded)
    return [b[:k] for b, k in zip(bufs, sizes)]
