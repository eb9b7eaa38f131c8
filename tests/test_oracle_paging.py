"""Pins of the oracle's paged-cache reading (``oracle.unpage``): row s of
sequence b lives at pool row table[b, s // page_size] * page_size +
s % page_size (paged key cache, section 3 of "Optimizing Inference for New
Model Architectures ...")."""
import numpy as np

import oracle
from indexed_sparse_attention_relu_b200 import workloads as W


def test_hand_worked_example():
    # pool of 3 pages x 2 rows; row r of the pool holds the value 10 * r
    pool = (10.0 * np.arange(6)).reshape(6, 1)
    table = np.array([[2, 0], [1, -1]])
    got = oracle.unpage(pool, table, page_size=2, Lmax=3)
    # sequence 0: s=0,1 on page 2 (pool rows 4, 5); s=2 on page 0 (pool row 0)
    # sequence 1: s=0,1 on page 1 (pool rows 2, 3); s=2 on an unused page -> 0
    want = np.array([[[40.0], [50.0], [0.0]],
                     [[20.0], [30.0], [0.0]]])
    assert np.array_equal(got, want)


def test_one_page_per_sequence_in_order_is_the_contiguous_layout():
    rng = np.random.default_rng(0)
    B, L, d = 3, 8, 4
    cache = rng.standard_normal((B, L, d))
    table = np.arange(B).reshape(B, 1)
    assert np.array_equal(oracle.unpage(cache.reshape(B * L, d), table, page_size=L, Lmax=L), cache)


def test_generated_layout_places_every_needed_page_once():
    lens = [100, 0, 300, 64, 1]
    table, num_pages = W.page_layout(lens, 300, 64, seed=7)
    used = table[table >= 0]
    assert len(used) == sum((n + 63) // 64 for n in lens) == num_pages - 3
    assert len(set(used.tolist())) == len(used) and used.max() < num_pages
    for b, n in enumerate(lens):
        assert np.all(table[b, :(n + 63) // 64] >= 0) and np.all(table[b, (n + 63) // 64:] == -1)
    # a pool whose row r holds r: unpage returns each needed row's pool position
    pool = np.arange(num_pages * 64, dtype=np.int64).reshape(-1, 1)
    logical = oracle.unpage(pool, table, 64, 300)[..., 0]
    for b, n in enumerate(lens):
        s = np.arange(n)
        assert np.array_equal(logical[b, :n], table[b, s // 64] * 64 + s % 64)
