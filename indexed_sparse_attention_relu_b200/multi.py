"""Host logic for running the decode hot path on several GPUs of one node.

Decode sequences are independent: every rank runs the whole path on its own
sequences and no data crosses GPUs. What remains on the host is

  * assigning sequences to ranks (longest first onto the least-loaded rank,
    so ragged context lengths do not leave one GPU with the long tail: the
    load skew of "later position, longer history" that the pages describe
    for causal work applies to ragged decode batches as well), and
  * timing: every rank times its own steps with CUDA events, and the job's
    time is the maximum over ranks (a job is done when its slowest rank is).

Both are plain functions of their inputs plus one all-reduce, so they run
under any torch.distributed backend (nccl on the GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import heapq
from typing import List, Sequence

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
