"""Multi-rank host logic on CPU: sequence sharding and max-over-ranks timing,
run as two gloo ranks (the same code path the benchmark takes on N GPUs with
the nccl backend; decode moves no data between GPUs)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from indexed_sparse_attention_relu_b200 import multi
from indexed_sparse_attention_relu_b200 import workloads as W


def test_shard_covers_every_sequence_once():
    rng = np.random.default_rng(3)
    lens = rng.integers(1024, 65537, 64)
    for world in (1, 2, 3, 4, 8):
        shards = multi.shard_sequences(lens, world)
        flat = sorted(b for s in shards for b in s)
        assert flat == list(range(len(lens)))
        assert all(s == sorted(s) for s in shards)


def test_shard_balance_is_within_one_sequence():
    """Greedy longest-first: the heaviest and lightest rank differ by at most
    the longest sequence (the classic bound of the LPT rule)."""
    rng = np.random.default_rng(7)
    for world in (2, 4, 8):
        lens = rng.integers(1024, 65537, 64)
        loads = multi.shard_loads(lens, multi.shard_sequences(lens, world))
        assert loads.sum() == lens.sum()
        assert loads.max() - loads.min() <= lens.max()


def test_shard_equal_lengths_split_evenly():
    shards = multi.shard_sequences([8192] * 32, 8)
    assert [len(s) for s in shards] == [4] * 8


def test_shard_ragged_decode_workload():
    """The ragged decode workload's own lengths (seed 3): 2 ranks within one
    sequence of each other."""
    wl = W.make("c3", with_caches=False)
    lens = wl.seq_lens.astype(np.int64)
    loads = multi.shard_loads(lens, multi.shard_sequences(lens, 2))
    assert abs(int(loads[0]) - int(loads[1])) <= int(lens.max())


def test_job_throughput_counts_all_ranks():
    assert multi.job_throughput([32, 32], 0.1) == pytest.approx(640000.0)
    with pytest.raises(ValueError):
        multi.job_throughput([1], 0.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # every rank derives the same assignment from the same lengths
        lens = [1000 + 37 * i for i in range(10)]
        shards = multi.shard_sequences(lens, world)
        mine = shards[rank]
        # per-rank "time" differs; the job time is the maximum
        local_ms = 1.0 + rank * 0.5
        job_ms = multi.max_over_ranks(local_ms, dist)
        units = torch.tensor([len(mine)], dtype=torch.int64)
        dist.all_reduce(units)
        q.put((rank, mine, job_ms, int(units.item())))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_agree():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got.sort()
    shards = [g[1] for g in got]
    assert sorted(shards[0] + shards[1]) == list(range(10))
    assert not set(shards[0]) & set(shards[1])
    assert all(g[2] == pytest.approx(1.5) for g in got)   # max over ranks
    assert all(g[3] == 10 for g in got)                    # every sequence counted once


def test_max_over_ranks_without_group_is_identity():
    assert multi.max_over_ranks(2.5) == 2.5
