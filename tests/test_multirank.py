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


# ----------------------------------------------------------------------------- zigzag context parallelism

def test_zigzag_matches_the_pages_examples():
    """The pages' two worked assignments: with 2 cards and 4 segments, card 0
    takes segments 1 and 4 and card 1 segments 2 and 3 (1-based); with 8
    devices... device 0 of a sequence of length L cut for 4 devices handles
    [0, L/8) and [7L/8, L)."""
    L = 4096
    two = multi.zigzag_segments(L, 2)
    seg = [(0, 1024), (1024, 2048), (2048, 3072), (3072, 4096)]
    assert two == [[seg[0], seg[3]], [seg[1], seg[2]]]
    four = multi.zigzag_segments(L, 4)
    assert four[0] == [(0, L // 8), (7 * L // 8, L)]


def test_zigzag_balances_causal_work():
    """Equal segments paired early-with-late give every rank the same causal
    work; a contiguous split gives the last rank 2N-1 times the first's."""
    T = 32768
    for world in (2, 4, 8):
        loads = [multi.causal_work(multi.zigzag_rows(T, world, d)) for d in range(world)]
        assert max(loads) == min(loads)
        assert sum(loads) == T * (T + 1) // 2
        contiguous = [multi.causal_work(np.arange(d * T // world, (d + 1) * T // world)) for d in range(world)]
        assert max(contiguous) / min(contiguous) > 2 * world - 1.5
    # uneven segment sizes (T not a multiple of 2N): within one segment's worth of rows
    T = 1001
    loads = [multi.causal_work(multi.zigzag_rows(T, 3, d)) for d in range(3)]
    assert max(loads) - min(loads) <= 2 * T


def test_zigzag_restore_is_the_inverse():
    rng = np.random.default_rng(5)
    for T, world in ((17, 2), (1000, 4), (64, 8), (3, 2)):
        data = rng.standard_normal((T, 3))
        parts = [data[multi.zigzag_rows(T, world, d)] for d in range(world)]
        assert np.array_equal(multi.zigzag_restore(parts, T, world), data)
        flat = np.sort(np.concatenate([multi.zigzag_rows(T, world, d) for d in range(world)]))
        assert np.array_equal(flat, np.arange(T))


def _cp_rank_main(rank, world, port, q):
    """One rank of a context-parallel prefill: it takes its zigzag rows, holds
    the cache rows of its own segments, all-gathers everyone's rows into the
    full caches, runs the whole path (the fp64 oracle stands in for the
    kernels on CPU) for its rows, and all-gathers the results."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import dataclasses
    import datetime

    import oracle

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = W.scaled("c4", B=1, Lmax=96, T_per_seq=96, K=16, HI=4, dI=32, H=4, dc=64, dr=16)
        rows = multi.zigzag_rows(wl.T, world, rank)
        # this rank's cache rows (positions = its query rows in a prefill)
        k_mine = torch.from_numpy(wl.k_idx[0, rows])
        kv_mine = torch.from_numpy(wl.kv[0, rows])
        pos_mine = torch.from_numpy(rows)
        k_all = multi.all_gather_rows(k_mine, dist)
        kv_all = multi.all_gather_rows(kv_mine, dist)
        pos_all = multi.all_gather_rows(pos_mine, dist)
        k_full = np.zeros_like(wl.k_idx)
        kv_full = np.zeros_like(wl.kv)
        for p, k, v in zip(pos_all, k_all, kv_all):
            k_full[0, p.numpy()] = k.numpy()
            kv_full[0, p.numpy()] = v.numpy()
        local = dataclasses.replace(wl, k_idx=k_full, kv=kv_full)
        _, idx, out, lse = oracle.dsa(local, rows)
        idx_all = multi.all_gather_rows(torch.from_numpy(idx), dist)
        out_all = multi.all_gather_rows(torch.from_numpy(out), dist)
        q.put((rank, [t.numpy() for t in idx_all], [t.numpy() for t in out_all]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_zigzag_context_parallel_prefill_two_gloo_ranks():
    """Two ranks reproduce the single-process result exactly once the zigzag
    shards are gathered and put back in order."""
    import oracle

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q.get(timeout=180) for _ in range(world)], key=lambda g: g[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    wl = W.scaled("c4", B=1, Lmax=96, T_per_seq=96, K=16, HI=4, dI=32, H=4, dc=64, dr=16)
    _, want_idx, want_out, _ = oracle.dsa(wl)
    for _, idx_parts, out_parts in got:           # every rank holds the whole result
        assert np.array_equal(multi.zigzag_restore(idx_parts, wl.T, world), want_idx)
        assert np.array_equal(multi.zigzag_restore(out_parts, wl.T, world), want_out)


def test_sharded_ragged_decode_covers_every_token_once():
    """bench.py --gpus N on the ragged decode gives each rank whole sequences
    (longest first, no exchange): every query token lands on exactly one rank,
    the per-rank workloads regenerate the same cache rows as the full batch,
    and the loads are balanced to within the longest sequence."""
    wl = W.make("c3", with_caches=False)
    for world in (2, 3, 8):
        shards = multi.shard_sequences(wl.seq_lens, world)
        parts = [W.select_sequences(wl, sh) for sh in shards]
        assert sum(p.T for p in parts) == wl.T
        seen = np.concatenate([p.seq_ids for p in parts])
        assert sorted(seen.tolist()) == list(range(wl.B))
        loads = [int(p.seq_lens.sum()) for p in parts]
        assert max(loads) - min(loads) <= int(wl.seq_lens.max())
    p = W.select_sequences(wl, [5, 17])
    assert np.array_equal(p.seq_rows("k_idx", 1), wl.seq_rows("k_idx", 17))
    assert np.array_equal(p.q_pos, wl.q_pos[[5, 17]])
