"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Sizes the oracle finishes in seconds that still span several tiles (128-key
indexer tiles, 64-key attention tiles) and a ragged tail, plus the edge cases
of the method (K >= context, K = 1, rows with fewer candidates than K, ties,
-1 padding, out-of-range indices). Full-size configurations are covered in
test_gpu_fullsize.py.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import device as DV
from indexed_sparse_attention_relu_b200 import workloads as W

from gpu_helpers import (check_attention, check_scores, check_topk_band, gpu_fused, gpu_mla, gpu_scores, gpu_topk,
                         oracle_codes, score_bound)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    """Every test starts and ends with a clean device status word."""
    B.dsa_read_device_status()
    yield


def _np(t):
    return t.cpu().numpy()


# ----------------------------------------------------------------------------- FP8 cache write

@pytest.mark.parametrize("group", [32, 64, 128])
def test_quantize_bit_exact(group):
    rng = np.random.default_rng(group)
    n, dim = 4099, 128
    k = (rng.standard_normal((n, dim)) * np.exp2(rng.integers(-20, 20, (n, 1)))).astype(np.float32)
    k[5] = 0.0                                    # all-zero key: scale 0, codes 0
    k[6, :] = 1e-38                               # tiny values (subnormal quotients)
    k[7, ::2] = -3.0e4
    k = W.bf16_round(k)
    codes, scales = oracle.quantize_keys(k, group)
    kt = DV.bf16_tensor(k, "cuda")
    k8 = torch.empty((n, dim), dtype=torch.uint8, device="cuda")
    sc = torch.empty((n, dim // group), dtype=torch.float32, device="cuda")
    B.dsa_quantize_index_keys(kt, group, k8, sc)
    assert np.array_equal(_np(sc), scales)
    assert np.array_equal(_np(k8), codes)
    deq = torch.empty((n, dim), dtype=torch.float32, device="cuda")
    B.dsa_dequantize_index_keys(k8, sc, group, deq)
    assert np.array_equal(_np(deq), oracle.dequantize_keys(codes, scales, group))


# ----------------------------------------------------------------------------- indexer

def test_indexer_c1_exact():
    wl = W.make("c1")
    dw = DV.to_device(wl)
    got = _np(gpu_scores(dw))
    want = oracle.indexer_scores(wl)
    nv = wl.n_valid()
    for t in range(wl.T):
        assert np.array_equal(got[t, :nv[t]], want[t, :nv[t]].astype(np.float32))
        assert np.all(got[t, nv[t]:] == -np.inf)


def _ragged_decode(name="c2", key_dtype=None, lens=(1000, 700, 129, 1), T_per_seq=1, K=256, integer=None):
    return W.scaled(name, B=len(lens), Lmax=max(lens) + 24, lens=lens, T_per_seq=T_per_seq, K=K,
                    key_dtype=key_dtype, integer=integer)


def test_indexer_bf16_ragged_decode():
    wl = _ragged_decode()
    dw = DV.to_device(wl)
    got = _np(gpu_scores(dw))
    want = oracle.indexer_scores(wl)
    check_scores(got, want, score_bound(wl), wl.n_valid())


def test_indexer_fp8_ragged_decode():
    wl = _ragged_decode(key_dtype="fp8")
    dw = DV.to_device(wl)
    codes, scales = oracle_codes(dw)
    got = _np(gpu_scores(dw))
    want = oracle.indexer_scores(wl, k_codes=codes, k_scales=scales)
    check_scores(got, want, score_bound(wl, k_codes=codes, k_scales=scales), wl.n_valid())


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("HI,dI", [(4, 32), (4, 128), (64, 32), (64, 128)])
def test_indexer_decode_shapes_integer_exact(HI, dI, key_dtype):
    """One query per sequence (the balanced decode kernel) for every supported
    indexer shape, integer values in [-2, 2] so every score is exact: BF16 keys
    give integer sums, FP8 keys give codes in {0, +-224, +-448} times one scale
    applied after the head sum (fl32 of an exact value)."""
    wl = W.scaled("c5i", B=5, Lmax=700, lens=(700, 129, 128, 1, 513), T_per_seq=1, K=64, HI=HI, dI=dI,
                  key_dtype=key_dtype, integer=True)
    dw = DV.to_device(wl)
    kw = {}
    if key_dtype == "fp8":
        codes, scales = oracle_codes(dw)
        kw = dict(k_codes=codes, k_scales=scales)
    got = _np(gpu_scores(dw))
    want = oracle.indexer_scores(wl, **kw)
    nv = wl.n_valid()
    for t in range(wl.T):
        assert np.array_equal(got[t, :nv[t]], want[t, :nv[t]].astype(np.float32)), t
        assert np.all(got[t, nv[t]:(nv[t] + 127) // 128 * 128] == -np.inf)


@pytest.mark.parametrize("Lmax", [1001, 1000])
def test_indexer_decode_fp8_scale_rows(Lmax):
    """FP8 decode: with max_seq_len a multiple of 4 every tile's 128 scales
    are copied into its stage (the last tile of the cache clipped at the end);
    otherwise each key's scale is read from global memory. Integer values:
    scores exact either way."""
    lens = (Lmax, 130, 1, Lmax - 3)
    wl = W.scaled("c5i", B=4, Lmax=Lmax, lens=lens, T_per_seq=1, K=64, HI=64, dI=128, key_dtype="fp8",
                  integer=True)
    dw = DV.to_device(wl)
    codes, scales = oracle_codes(dw)
    got = _np(gpu_scores(dw))
    want = oracle.indexer_scores(wl, k_codes=codes, k_scales=scales)
    nv = wl.n_valid()
    for t in range(wl.T):
        assert np.array_equal(got[t, :nv[t]], want[t, :nv[t]].astype(np.float32)), t


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_indexer_decode_ranges_span_many_tokens(key_dtype):
    """200 short sequences (one of them empty): the flattened key-tile list has
    fewer tiles than twice the CTA count, so CTA ranges start and end inside
    tokens and run across several of them."""
    rng = np.random.default_rng(21)
    lens = rng.integers(1, 400, 200)
    lens[17] = 0
    wl = W.scaled("c2", B=200, Lmax=400, lens=tuple(int(x) for x in lens), T_per_seq=1, K=128, key_dtype=key_dtype)
    dw = DV.to_device(wl)
    kw = {}
    if key_dtype == "fp8":
        codes, scales = oracle_codes(dw)
        kw = dict(k_codes=codes, k_scales=scales)
    got = _np(gpu_scores(dw))
    want = oracle.indexer_scores(wl, **kw)
    check_scores(got, want, score_bound(wl, **kw), wl.n_valid())


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_indexer_causal_prefill_groups(key_dtype):
    """Several tokens per sequence: the 4-token MMA groups, causal masks that
    differ inside a group, and groups that end mid-sequence."""
    wl = W.scaled("c4", B=2, Lmax=700, lens=(700, 333), T_per_seq=150, K=128, key_dtype=key_dtype)
    dw = DV.to_device(wl)
    got = _np(gpu_scores(dw))
    if key_dtype == "fp8":
        codes, scales = oracle_codes(dw)
        want = oracle.indexer_scores(wl, k_codes=codes, k_scales=scales)
        bound = score_bound(wl, k_codes=codes, k_scales=scales)
    else:
        want = oracle.indexer_scores(wl)
        bound = score_bound(wl)
    check_scores(got, want, bound, wl.n_valid())


def test_indexer_integer_fp8_exact():
    """Integer values in [-2, 2]: FP8 codes are {0, +-224, +-448}, every partial
    sum is an integer below 2^24, so the kernel's score is fl32(scale * N) with
    N exact -- equal to the oracle's exact fp64 score rounded once to fp32."""
    wl = W.scaled("c5i", B=2, Lmax=600, lens=(600, 257), T_per_seq=5, K=64, key_dtype="fp8", integer=True)
    dw = DV.to_device(wl)
    codes, scales = oracle_codes(dw)
    got = _np(gpu_scores(dw))
    want = oracle.indexer_scores(wl, k_codes=codes, k_scales=scales)
    nv = wl.n_valid()
    for t in range(wl.T):
        assert np.array_equal(got[t, :nv[t]], want[t, :nv[t]].astype(np.float32)), t


# ----------------------------------------------------------------------------- top-k

def test_topk_bit_exact_on_kernel_scores():
    """Given the kernel's own fp32 scores, the selection is fully determined:
    the oracle's sort on the same values must give identical indices."""
    wl = _ragged_decode(lens=(1000, 700, 129, 1, 5000), K=256)
    dw = DV.to_device(wl)
    sc = gpu_scores(dw)
    idx = _np(gpu_topk(dw, sc))
    want = oracle.topk(_np(sc).astype(np.float64), wl.n_valid(), wl.K)
    assert np.array_equal(idx, want)


def _topk_rows(rows, K):
    """Run the kernel on hand-built score rows (one sequence per row)."""
    n = len(rows)
    L = max(len(r) for r in rows)
    sc = np.full((n, L), -np.inf, np.float32)
    for i, r in enumerate(rows):
        sc[i, :len(r)] = r
    lens = np.array([len(r) for r in rows], np.int32)
    batch = B.Batch(torch.arange(n + 1, dtype=torch.int32, device="cuda"),
                    torch.from_numpy(lens - 1).cuda(), torch.from_numpy(lens).cuda(), L)
    st = torch.from_numpy(sc).cuda()
    idx = torch.full((n, K), -7, dtype=torch.int32, device="cuda")
    B.dsa_topk(batch, st, K, idx)
    torch.cuda.synchronize()
    return _np(idx), sc, lens


def test_topk_tie_cases():
    K = 64
    rows = [
        np.zeros(300, np.float32),                                  # all equal: first K positions
        np.where(np.arange(200) % 2 == 0, -0.0, 0.0).astype(np.float32),  # -0 ties +0
        np.arange(40, dtype=np.float32),                            # fewer than K: all, -1 padded
        np.repeat(np.arange(10, dtype=np.float32), 30),             # long tie runs at the threshold
        np.float32(np.random.default_rng(1).integers(-3, 4, 5000)),  # many ties, long row
    ]
    idx, sc, lens = _topk_rows(rows, K)
    want = oracle.topk(sc.astype(np.float64), lens, K)
    assert np.array_equal(idx, want)
    assert list(idx[0]) == list(range(K))
    assert list(idx[2][:40]) == list(range(40)) and np.all(idx[2][40:] == -1)


def test_topk_register_rows_full_and_ragged():
    """Rows held in registers: 8192 positions (8 keys a thread, aligned
    vector loads, the decode shape with K = 2048) and up to 16383 positions
    (16 keys a thread; an odd row stride leaves rows unaligned, so keys load
    one at a time), with ties at the threshold and an all-equal row."""
    rng = np.random.default_rng(11)
    full = [W.bf16_round(rng.standard_normal(8192).astype(np.float32) * 8),
            np.float32(rng.integers(-20, 20, 8192)),
            np.zeros(8192, np.float32)]
    idx, sc, lens = _topk_rows(full, 2048)
    assert np.array_equal(idx, oracle.topk(sc.astype(np.float64), lens, 2048))
    assert list(idx[2]) == list(range(2048))
    ragged = [W.bf16_round(rng.standard_normal(16383).astype(np.float32) * 8),
              np.float32(rng.integers(-20, 20, 12001)),
              np.zeros(9000, np.float32),
              W.bf16_round(rng.standard_normal(2049).astype(np.float32)),
              np.float32(rng.integers(0, 3, 1500))]
    idx, sc, lens = _topk_rows(ragged, 2048)
    assert np.array_equal(idx, oracle.topk(sc.astype(np.float64), lens, 2048))


@pytest.mark.parametrize("L", [8192, 16384, 32768, 65536])
def test_topk_threshold_ties_at_each_kernel_limit(L):
    """Rows of 8192 and 16384 positions (held in registers) and of 32768 and
    65536 (position bitmaps and a candidate list in shared memory), each at
    the longest row of its kernel: an all-equal row, integer scores and a few
    large values over a constant bulk put long runs of ties at the threshold,
    across thread and chunk boundaries; a shorter row and one of fewer than K
    positions ride along in the same launch."""
    rng = np.random.default_rng(L)
    bulk = np.full(L, 0.5, np.float32)
    bulk[rng.choice(L, 1500, replace=False)] = 3.0
    rows = [np.zeros(L, np.float32),
            np.float32(rng.integers(-4, 5, L)),
            bulk,
            W.bf16_round(rng.standard_normal(L).astype(np.float32) * 8),
            W.bf16_round(rng.standard_normal(L // 2 + 3).astype(np.float32)),
            np.float32(rng.integers(0, 2, 2000))]
    idx, sc, lens = _topk_rows(rows, 2048)
    assert np.array_equal(idx, oracle.topk(sc.astype(np.float64), lens, 2048))
    assert list(idx[0]) == list(range(2048))


def test_topk_streaming_rows_unaligned():
    """Rows above 16384 positions stream from memory; an odd row stride leaves
    all but the first row unaligned (positions load one at a time) and the
    lengths leave ragged ends after the last whole group of four."""
    rng = np.random.default_rng(13)
    rows = [W.bf16_round(rng.standard_normal(20001).astype(np.float32) * 8),
            W.bf16_round(rng.standard_normal(17003).astype(np.float32) * 8),
            np.float32(rng.integers(-30, 30, 18002)),
            W.bf16_round(rng.standard_normal(16385).astype(np.float32))]
    idx, sc, lens = _topk_rows(rows, 2048)
    assert np.array_equal(idx, oracle.topk(sc.astype(np.float64), lens, 2048))


def test_topk_long_rows_and_crowded_threshold_bin():
    """Long rows (two streaming passes), and rows whose threshold bin holds more
    keys than the candidate list (all equal, or a constant bulk under a few
    larger values): the exact threshold is then found by streaming the row
    restricted to that bin."""
    rng = np.random.default_rng(7)
    bulk = np.full(60_000, 0.75, np.float32)
    bulk[rng.choice(60_000, 1000, replace=False)] = 2.0
    rows = [W.bf16_round(rng.standard_normal(70_000).astype(np.float32) * 8),
            np.float32(rng.integers(-50, 50, 60_000)),
            np.zeros(60_000, np.float32),
            bulk]
    idx, sc, lens = _topk_rows(rows, 2048)
    want = oracle.topk(sc.astype(np.float64), lens, 2048)
    assert np.array_equal(idx, want)
    assert list(idx[2]) == list(range(2048))


def test_topk_rows_beyond_the_bitmap_budget():
    """Rows so long (800 000 positions) that two position bitmaps no longer fit
    in shared memory: the one-pass-per-digit radix kernel streams the row from
    memory for each 8-bit digit."""
    rng = np.random.default_rng(17)
    rows = [W.bf16_round(rng.standard_normal(800_000).astype(np.float32) * 8),
            np.float32(rng.integers(-40, 40, 790_001))]
    idx, sc, lens = _topk_rows(rows, 2048)
    assert np.array_equal(idx, oracle.topk(sc.astype(np.float64), lens, 2048))


# ----------------------------------------------------------------------------- sparse MLA

def _mla_check(wl, idx_np):
    dw = DV.to_device(wl)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    out, lse = gpu_mla(dw, idx)
    want_out, want_lse = oracle.sparse_mla(wl, idx_np)
    return check_attention(out, lse, want_out, want_lse)


@pytest.mark.parametrize("T_per_seq,H", [(1, 128), (16, 128), (40, 128), (1, 64), (40, 64)])
def test_mla_matches_oracle(T_per_seq, H):
    """128 heads (score CTA + value CTA pairs): T_per_seq=1 -> 2 queries, 3
    key splits (a cluster of 6 CTAs, merged through the workspace); 16 -> 32
    queries, split in 2; 40 -> 80 queries, one split each. 64 heads (one CTA
    per head block): the same split regimes. K=300 leaves a ragged 64-key
    tail and -1 padding."""
    wl = W.scaled("c2", B=2, Lmax=900, lens=(900, 400), T_per_seq=T_per_seq, K=300, H=H)
    rng = np.random.default_rng(T_per_seq)
    nv = wl.n_valid()
    idx = np.full((wl.T, wl.K), -1, np.int32)
    for t in range(wl.T):
        m = min(wl.K - 7, nv[t])
        idx[t, :m] = rng.choice(nv[t], m, replace=False)
        rng.shuffle(idx[t])
    _mla_check(wl, idx)


def test_mla_small_latent_c1_shapes():
    wl = W.make("c1")
    sc = oracle.indexer_scores(wl)
    idx = oracle.topk(sc, wl.n_valid(), wl.K)
    _mla_check(wl, idx)


def test_mla_many_tiles_per_split():
    """Many queries -> one key split per query with several 64-key tiles each
    (the pipelined gather / PV / QK^T order), plus the lazy-rescale path: every
    head's query gets 8 in its first rope dim and the keys at positions >= 600
    get 32 there (0 before), so later tiles' logits rise uniformly by
    8 * 32 / sqrt(576) = 10.7 (15.4 in log2 units, above the 2^8 rescale
    threshold) while the softmax over them stays as flat as before."""
    wl = W.scaled("c2", B=1, Lmax=1200, lens=(1200,), T_per_seq=160, K=640)
    q = wl.q.copy()
    kv = wl.kv.copy()
    q[:, :, wl.dc] = 8.0
    kv[0, :600, wl.dc] = 0.0
    kv[0, 600:1200, wl.dc] = 32.0
    wl = dataclasses.replace(wl, kv=kv, q=q)
    nv = wl.n_valid()
    idx = np.full((wl.T, wl.K), -1, np.int32)
    for t in range(wl.T):
        m = min(wl.K, nv[t])
        idx[t, :m] = np.arange(nv[t] - m, nv[t])        # ascending: small logits first
    _mla_check(wl, idx)


def test_mla_dense_when_k_covers_context():
    wl = W.scaled("c2", B=1, Lmax=200, lens=(200,), T_per_seq=3, K=256)
    nv = wl.n_valid()
    idx = np.full((wl.T, wl.K), -1, np.int32)
    for t in range(wl.T):
        idx[t, :nv[t]] = np.arange(nv[t])
    _mla_check(wl, idx)


def test_mla_single_key_is_value_row():
    wl = W.scaled("c2", B=2, Lmax=100, lens=(100, 50), T_per_seq=2, K=64)
    idx = np.full((wl.T, wl.K), -1, np.int32)
    pick = [99, 3, 0, 49]
    for t in range(wl.T):
        idx[t, 17] = pick[t]
    dw = DV.to_device(wl)
    out, lse = gpu_mla(dw, torch.from_numpy(idx).cuda())
    b = wl.seq_of_token()
    o = _np(out.float())
    for t in range(wl.T):
        row = wl.kv[b[t], pick[t], :wl.dc]
        assert np.array_equal(o[t], np.broadcast_to(row, o[t].shape))   # bf16 value reproduced exactly


def test_mla_out_of_range_indices_are_skipped_and_flagged():
    wl = W.scaled("c2", B=1, Lmax=300, lens=(300,), T_per_seq=2, K=64)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(300, 64, replace=False) for _ in range(wl.T)]).astype(np.int32)
    bad = idx.copy()
    bad[0, 5] = 300          # == seq_len: out of range
    bad[1, 9] = 10_000_000
    bad[1, 10] = -5
    dw = DV.to_device(wl)
    out, lse = gpu_mla(dw, torch.from_numpy(bad).cuda(), expect_status_ok=False)
    assert B.dsa_read_device_status() == B.DSA_ERR_DEVICE_INDEX
    assert B.dsa_read_device_status() == B.DSA_OK            # sticky until read, then clear
    clean = bad.copy()
    clean[(clean < 0) | (clean >= 300)] = -1
    want_out, want_lse = oracle.sparse_mla(wl, clean)
    check_attention(out, lse, want_out, want_lse)


# ----------------------------------------------------------------------------- whole chain

def test_fused_decode_c1_bit_exact_indices():
    wl = W.make("c1")
    dw = DV.to_device(wl)
    out, lse, idx = gpu_fused(dw)
    sc, want_idx, want_out, want_lse = oracle.dsa(wl)
    assert np.array_equal(_np(idx), want_idx)
    check_attention(out, lse, want_out, want_lse)
    assert B.dsa_read_device_status() == B.DSA_OK


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_fused_decode_ragged(key_dtype):
    wl = _ragged_decode(key_dtype=key_dtype, lens=(3000, 1100, 2048, 77), K=2048)
    dw = DV.to_device(wl)
    out, lse, idx = gpu_fused(dw)
    kw = {}
    if key_dtype == "fp8":
        codes, scales = oracle_codes(dw)
        kw = dict(k_codes=codes, k_scales=scales)
    sc = oracle.indexer_scores(wl, **kw)
    want_idx = oracle.topk(sc, wl.n_valid(), wl.K)
    check_topk_band(_np(idx), want_idx, sc, wl.K)
    # attention checked on the kernel's own selection
    want_out, want_lse = oracle.sparse_mla(wl, _np(idx))
    check_attention(out, lse, want_out, want_lse)
    assert B.dsa_read_device_status() == B.DSA_OK


def test_fused_decode_is_deterministic():
    wl = _ragged_decode(lens=(2500, 900), K=512)
    dw = DV.to_device(wl)
    a = gpu_fused(dw)
    b = gpu_fused(dw)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.uint8) if y.dtype == torch.bfloat16 else y)
