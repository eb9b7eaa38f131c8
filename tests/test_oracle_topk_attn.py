"""Pins for the oracle's Top-K and sparse MLA attention.

Top-K (Lightning Indexer selection, section 1 of "Day-0 Inference Optimization
for a New Sparse Attention Architecture") is pinned by a characterisation that
needs no sort: the selected set S has size min(K, n) and is upper-closed under
the order (score desc, position asc), i.e. every selected position beats every
unselected one. Hand-built tie cases fix the tie rule.

Sparse attention (Sparse Flash Attention over MLA rows, same section) is pinned
by special cases that reduce to other computations: K >= context is dense
causal attention (numpy matmul + scipy softmax); K = 1 returns the value row;
two keys give the logistic closed form; constant values are reproduced
exactly (weights sum to one); outputs lie in the convex hull of the selected
values; the order of the indices and -1 padding do not matter.
"""
import dataclasses

import numpy as np
import pytest
import scipy.special

import oracle
from indexed_sparse_attention_relu_b200 import workloads as W


# ----------------------------------------------------------------------------- top-k

def _beats(sa, ia, sb, ib):
    return sa > sb or (sa == sb and ia < ib)


def _check_selection(scores, nv, K, idx):
    n = int(nv)
    take = min(K, n)
    sel = [int(i) for i in idx if i >= 0]
    assert len(sel) == take
    assert all(i == -1 for i in idx[take:])
    assert sel == sorted(sel) and len(set(sel)) == take
    assert all(0 <= i < n for i in sel)
    chosen = set(sel)
    for i in chosen:
        for j in range(n):
            if j not in chosen:
                assert _beats(scores[i], i, scores[j], j), (i, j)


def test_topk_characterisation_random_rows():
    rng = np.random.default_rng(2)
    for trial in range(60):
        n = int(rng.integers(1, 40))
        K = int(rng.integers(1, 12))
        L = n + int(rng.integers(0, 5))
        row = np.full(L, -np.inf)
        # few distinct values -> many ties
        row[:n] = rng.integers(-3, 4, n).astype(np.float64) * (0.5 if trial % 2 else 1.0)
        idx = oracle.topk(row[None], [n], K)[0]
        _check_selection(row, n, K, idx)


def test_topk_brute_force_tiny_rows():
    """Exhaustive: over all subsets of size K, the chosen one is the unique
    upper-closed subset."""
    import itertools
    rng = np.random.default_rng(3)
    for _ in range(30):
        n = int(rng.integers(1, 9))
        K = int(rng.integers(1, n + 1))
        row = rng.integers(-2, 3, n).astype(np.float64)
        good = [c for c in itertools.combinations(range(n), K)
                if all(_beats(row[i], i, row[j], j) for i in c for j in range(n) if j not in c)]
        assert len(good) == 1
        idx = oracle.topk(row[None], [n], K)[0]
        assert tuple(idx) == good[0]


def test_topk_tie_cases():
    # all equal -> the first K positions
    row = np.zeros((1, 10))
    assert list(oracle.topk(row, [10], 4)[0]) == [0, 1, 2, 3]
    # -0 ties with +0; lower position wins
    row = np.array([[-0.0, 1.0, 0.0, -1.0]])
    assert list(oracle.topk(row, [4], 2)[0]) == [0, 1]
    # fewer valid than K: all valid, padded with -1; entries past n_valid ignored
    row = np.array([[5.0, 1.0, 9.0, 100.0, 100.0]])
    assert list(oracle.topk(row, [3], 5)[0]) == [0, 1, 2, -1, -1]
    # -inf inside the row beyond n_valid never selected
    row = np.array([[1.0, -np.inf, -np.inf]])
    assert list(oracle.topk(row, [1], 3)[0]) == [0, -1, -1]


# ----------------------------------------------------------------------------- attention

def _mla_case(seed=0, B=2, L=50, H=3, dc=8, dr=4, T_per=(2, 1), lens=(50, 31)):
    rng = np.random.default_rng(seed)
    T = sum(T_per)
    cu = np.concatenate([[0], np.cumsum(T_per)]).astype(np.int32)
    D = dc + dr
    kv = W.bf16_round(rng.standard_normal((B, L, D)).astype(np.float32))
    for b in range(B):
        kv[b, lens[b]:] = 0
    q = W.bf16_round(rng.standard_normal((T, H, D)).astype(np.float32))
    b_of = np.searchsorted(cu, np.arange(T), side="right") - 1
    pos = np.array([lens[b] - 1 - i for i, b in enumerate(b_of)], np.int32)
    return W.Workload(name="pin", B=B, T=T, Lmax=L, cu_q=cu, q_pos=pos, seq_lens=np.array(lens, np.int32),
                      HI=1, dI=1, H=H, dc=dc, dr=dr, K=L, key_dtype="bf16", scale_group=1,
                      softmax_scale=float(1 / np.sqrt(D)), q_idx=np.zeros((T, 1, 1), np.float32),
                      w=np.zeros((T, 1), np.float32), k_idx=np.zeros((B, L, 1), np.float32), q=q, kv=kv,
                      seed=seed, integer_valued=False)


def test_full_selection_equals_dense_causal_attention():
    wl = _mla_case()
    nv = wl.n_valid()
    K = wl.Lmax
    idx = np.full((wl.T, K), -1, np.int32)
    for t in range(wl.T):
        idx[t, :nv[t]] = np.arange(nv[t])
    out, lse = oracle.sparse_mla(wl, idx)
    b_of = wl.seq_of_token()
    for t in range(wl.T):
        kvb = wl.kv[b_of[t], :nv[t]].astype(np.float64)
        z = (wl.q[t].astype(np.float64) @ kvb.T) * wl.softmax_scale          # [H, n]
        p = scipy.special.softmax(z, axis=-1)
        np.testing.assert_allclose(out[t], p @ kvb[:, :wl.dc], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[t], scipy.special.logsumexp(z, axis=-1), rtol=1e-12, atol=1e-12)


def test_single_key_returns_value_row_exactly():
    wl = _mla_case(seed=1)
    # make the rope part large and distinct so a wrong value slice would show
    wl.kv[..., wl.dc:] = 1000.0
    idx = np.full((wl.T, 5), -1, np.int32)
    b_of = wl.seq_of_token()
    pick = [7, 3, 0]
    for t in range(wl.T):
        idx[t, 2] = pick[t]
    out, lse = oracle.sparse_mla(wl, idx)
    for t in range(wl.T):
        row = wl.kv[b_of[t], pick[t]].astype(np.float64)
        assert np.array_equal(out[t], np.broadcast_to(row[:wl.dc], out[t].shape))
        np.testing.assert_allclose(lse[t], wl.softmax_scale * (wl.q[t].astype(np.float64) @ row), rtol=1e-13)


def test_two_keys_logistic_closed_form():
    wl = _mla_case(seed=2)
    b_of = wl.seq_of_token()
    idx = np.full((wl.T, 4), -1, np.int32)
    idx[:, 0], idx[:, 3] = 1, 4
    out, lse = oracle.sparse_mla(wl, idx)
    for t in range(wl.T):
        v1 = wl.kv[b_of[t], 1].astype(np.float64)
        v2 = wl.kv[b_of[t], 4].astype(np.float64)
        q = wl.q[t].astype(np.float64)
        z1, z2 = wl.softmax_scale * (q @ v1), wl.softmax_scale * (q @ v2)
        a = 1.0 / (1.0 + np.exp(-(z1 - z2)))
        np.testing.assert_allclose(out[t], a[:, None] * v1[:wl.dc] + (1 - a)[:, None] * v2[:wl.dc], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[t], np.logaddexp(z1, z2), rtol=1e-13)


def test_constant_values_and_convex_hull_and_permutation():
    wl = _mla_case(seed=3)
    rng = np.random.default_rng(4)
    b_of = wl.seq_of_token()
    nv = wl.n_valid()
    K = 9
    idx = np.stack([np.sort(rng.choice(nv[t], K, replace=False)) for t in range(wl.T)]).astype(np.int32)
    out, lse = oracle.sparse_mla(wl, idx)
    for t in range(wl.T):
        V = wl.kv[b_of[t], idx[t], :wl.dc].astype(np.float64)
        assert np.all(out[t] >= V.min(0) - 1e-12) and np.all(out[t] <= V.max(0) + 1e-12)
    # permuted order and interleaved -1 padding: identical result
    perm = np.stack([rng.permutation(K) for _ in range(wl.T)])
    idx2 = np.take_along_axis(idx, perm, 1)
    idx2 = np.concatenate([idx2, np.full((wl.T, 3), -1, np.int32)], 1)[:, rng.permutation(K + 3)]
    out2, lse2 = oracle.sparse_mla(wl, idx2)
    np.testing.assert_allclose(out2, out, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13)
    # constant value rows are reproduced exactly: the weights sum to one
    kv = wl.kv.copy()
    kv[..., :wl.dc] = np.float32(0.375)
    out3, _ = oracle.sparse_mla(dataclasses.replace(wl, kv=kv), idx)
    np.testing.assert_allclose(out3, 0.375, rtol=1e-14)


def test_no_valid_key_gives_zero_and_minus_inf():
    wl = _mla_case(seed=5)
    idx = np.full((wl.T, 3), -1, np.int32)
    idx[0, 1] = 10_000          # out of range: skipped
    out, lse = oracle.sparse_mla(wl, idx)
    assert not out.any() and np.all(lse == -np.inf)


def test_c1_end_to_end_is_integer_exact_through_topk():
    """Config 1 (integer values): scores are exact, so index selection is fully
    determined; the selection satisfies the characterisation."""
    wl = W.make("c1")
    sc, idx, out, lse = oracle.dsa(wl)
    nv = wl.n_valid()
    for t in range(wl.T):
        _check_selection(sc[t], nv[t], wl.K, idx[t])


def test_c1_matches_stored_golden():
    """Guards the oracle against silent change: the stored C1 expectation was
    written by tests/golden/make_golden.py from the oracle alone."""
    import json
    import os
    doc = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "c1_expected.json")))
    wl = W.make("c1")
    sc, idx, out, lse = oracle.dsa(wl)
    nv = wl.n_valid()
    for t in range(wl.T):
        assert [int(v) for v in sc[t, :nv[t]]] == doc["scores"][t]
    assert idx.tolist() == doc["idx"]
    want = np.array([[[float.fromhex(x) for x in h] for h in t] for t in doc["out"]])
    np.testing.assert_allclose(out, want, rtol=1e-14, atol=1e-14)
    want_lse = np.array([[float.fromhex(x) for x in t] for t in doc["lse"]])
    np.testing.assert_allclose(lse, want_lse, rtol=1e-14)
