"""Pins for the oracle's Lightning Indexer scores.

Score law: I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:]) over the causal
history s <= pos(t), s < len(seq) (scoring, head-weight weighting: section 3 of
"Optimizing Inference for New Model Architectures ..."; "later position =
longer history": its section 1 item 3).

The oracle is pinned by identities of the mathematics, not by a retyped copy:
since max(0, x) = (x + |x|) / 2, the scores for q and -q satisfy
    I(q) - I(-q) = sum_j w_j (q_j . k)     (a plain matrix product)
    I(q) + I(-q) = sum_j w_j |q_j . k|
which numpy's matmul evaluates independently; together they fix I exactly,
including where the ReLU sits and which operand each index runs over.
"""
import dataclasses

import numpy as np

import oracle
from indexed_sparse_attention_relu_b200 import workloads as W


def _small(seed=3, B=3, L=37, HI=5, dI=7, T_per=(3, 1, 2), lens=(37, 20, 9), integer=False):
    rng = np.random.default_rng(seed)
    T = sum(T_per)
    cu = np.concatenate([[0], np.cumsum(T_per)]).astype(np.int32)
    pos = np.concatenate([np.sort(rng.choice(np.arange(0, L + 5), n, replace=False)) for n in T_per]).astype(np.int32)
    if integer:
        dr = lambda *s: rng.integers(-3, 4, s).astype(np.float32)
    else:
        dr = lambda *s: W.bf16_round(rng.standard_normal(s).astype(np.float32))
    kI = dr(B, L, dI)
    for b in range(B):
        kI[b, lens[b]:] = 0
    return W.Workload(name="pin", B=B, T=T, Lmax=L, cu_q=cu, q_pos=pos, seq_lens=np.array(lens, np.int32),
                      HI=HI, dI=dI, H=1, dc=1, dr=0, K=4, key_dtype="bf16", scale_group=dI, softmax_scale=1.0,
                      q_idx=dr(T, HI, dI), w=dr(T, HI), k_idx=kI, q=np.zeros((T, 1, 1), np.float32),
                      kv=np.zeros((B, L, 1), np.float32), seed=seed, integer_valued=integer)


def test_relu_identities_pin_scores():
    wl = _small()
    neg = dataclasses.replace(wl, q_idx=-wl.q_idx)
    Ip = oracle.indexer_scores(wl)
    In = oracle.indexer_scores(neg)
    b = wl.seq_of_token()
    nv = wl.n_valid()
    for t in range(wl.T):
        kb = wl.k_idx[b[t]].astype(np.float64)                   # [L, dI]
        dots = wl.q_idx[t].astype(np.float64) @ kb.T            # [HI, L]
        lin = wl.w[t].astype(np.float64) @ dots                 # sum_j w_j (q_j . k)
        absd = wl.w[t].astype(np.float64) @ np.abs(dots)        # sum_j w_j |q_j . k|
        v = slice(0, nv[t])
        np.testing.assert_allclose(Ip[t, v] - In[t, v], lin[v], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(Ip[t, v] + In[t, v], absd[v], rtol=1e-12, atol=1e-12)


def test_causal_and_length_mask():
    wl = _small()
    I = oracle.indexer_scores(wl)
    b = wl.seq_of_token()
    for t in range(wl.T):
        nv = min(wl.q_pos[t] + 1, wl.seq_lens[b[t]])
        assert np.all(np.isfinite(I[t, :nv]))
        assert np.all(I[t, nv:] == -np.inf)
        # the query's own position is part of its history (when inside the cache)
        if wl.q_pos[t] < wl.seq_lens[b[t]]:
            assert np.isfinite(I[t, wl.q_pos[t]])


def test_linear_in_w_and_head_permutation():
    wl = _small(seed=4)
    rng = np.random.default_rng(0)
    w2 = rng.standard_normal(wl.w.shape).astype(np.float32)
    I1 = oracle.indexer_scores(wl)
    I2 = oracle.indexer_scores(dataclasses.replace(wl, w=w2))
    I12 = oracle.indexer_scores(dataclasses.replace(wl, w=(wl.w.astype(np.float64) + w2).astype(np.float32)))
    fin = np.isfinite(I1)
    # w and w2 are small-integer free floats; sum may round in fp32, so compare loosely
    np.testing.assert_allclose(I12[fin], (I1 + I2)[fin], rtol=1e-5, atol=1e-5)
    perm = rng.permutation(wl.HI)
    Ip = oracle.indexer_scores(dataclasses.replace(wl, q_idx=wl.q_idx[:, perm], w=wl.w[:, perm]))
    np.testing.assert_allclose(Ip[fin], I1[fin], rtol=1e-12, atol=1e-12)


def test_integer_inputs_give_exact_integers():
    wl = W.make("c1")
    I = oracle.indexer_scores(wl)
    fin = np.isfinite(I)
    assert np.array_equal(I[fin], np.round(I[fin]))
    assert np.abs(I[fin]).max() <= 4 * 3 * 32 * 9


def test_fp8_keys_equal_bf16_path_on_exact_dequantisation():
    """FP8 keys with power-of-two scales dequantise exactly in fp32, so the
    FP8 path must equal the plain path run on those dequantised keys."""
    wl = _small(seed=9, dI=8)
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 256, size=wl.k_idx.shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x10                       # no NaN codes
    scales = np.exp2(rng.integers(-3, 4, size=wl.k_idx.shape[:-1] + (1,))).astype(np.float32)
    deq = (oracle.e4m3_decode(codes) * scales).astype(np.float32)
    assert np.array_equal(deq.astype(np.float64), oracle.e4m3_decode(codes) * scales)
    I8 = oracle.indexer_scores(wl, k_codes=codes, k_scales=scales)
    Ib = oracle.indexer_scores(dataclasses.replace(wl, k_idx=deq))
    assert np.array_equal(I8, Ib)


def test_all_negative_dots_give_zero_scores():
    """Non-negative query heads against non-positive keys: every dot is <= 0,
    so the ReLU zeroes every head whatever the sign of w."""
    wl = _small(seed=12)
    q = np.abs(wl.q_idx) + np.float32(0.5)
    k = -np.abs(wl.k_idx) - np.float32(0.25)
    for b in range(wl.B):
        k[b, wl.seq_lens[b]:] = 0
    I = oracle.indexer_scores(dataclasses.replace(wl, q_idx=W.bf16_round(q), k_idx=W.bf16_round(k)))
    fin = np.isfinite(I)
    assert fin.any() and np.all(I[fin] == 0.0)
