"""Host-side accounting of the benchmark: the algorithmic bytes behind every
roofline figure, checked against the byte counts of the decode workload worked
out by hand (32 sequences of 8192 positions, one query each, K = 2048)."""
import numpy as np

import bench
from indexed_sparse_attention_relu_b200 import workloads as W


def test_decode_algorithmic_bytes_by_hand():
    wl = W.make("c2", with_caches=False)
    n_sel = int(np.minimum(wl.n_valid(), wl.K).sum())
    assert n_sel == 32 * 2048
    a = bench.algorithmic_bytes(wl, n_sel)
    keys = 32 * 8192 * 128 * 2                 # BF16 index keys, every causal candidate once
    q_i = 32 * 64 * 128 * 2
    w = 32 * 64 * 4
    scores = 32 * 8192 * 4                     # fp32 score rows
    rows = 32 * 2048 * 576 * 2                 # gathered latent rows
    q = 32 * 128 * 576 * 2
    idx = 32 * 2048 * 4
    out = 32 * 128 * 512 * 2
    assert (keys, rows, q, out, q_i, w) == (67108864, 75497472, 4718592, 4194304, 524288, 8192)
    assert a["indexer"] == keys + q_i + w + scores
    assert a["topk"] == scores + idx
    assert a["sparse_mla"] == rows + q + idx + out == 84672512
    assert a["step"] == keys + q_i + w + rows + q + idx + out == 152313856


def test_fp8_keys_count_codes_and_scales():
    """FP8 index keys move one byte per element plus one fp32 scale per key."""
    wl = W.make("c3", with_caches=False)
    a = bench.algorithmic_bytes(wl, int(np.minimum(wl.n_valid(), wl.K).sum()))
    rows = int(wl.seq_lens.astype(np.int64).sum())   # one query per sequence at its last position
    scores = int(wl.n_valid().astype(np.int64).sum()) * 4
    assert a["indexer"] == rows * (128 + 4) + wl.T * wl.HI * wl.dI * 2 + wl.T * wl.HI * 4 + scores


def test_cpu_baseline_repeats_until_the_minimum_time():
    wl = W.make("c1", with_caches=False)
    n, dt, thr = bench.run_cpu_oracle(wl, 2, min_seconds=0.2)
    assert dt >= 0.2 and n % 2 == 0 and n >= 2 and thr >= 1


def test_prefill_flops_by_hand():
    """Causal prefill of 32768 tokens: the indexer scores every causal pair
    (sum_{t<32768} (t+1) pairs) at 64 heads x 128 dims, and the attention runs
    QK^T over 576 dims and PV over 512 dims for min(t+1, 2048) selected rows
    per token at 128 heads. (Shapes only: the query tensors are not drawn.)"""
    import types
    nv = np.arange(1, 32769, dtype=np.int32)
    wl = types.SimpleNamespace(HI=64, dI=128, H=128, D=576, dc=512, K=2048, n_valid=lambda: nv)
    n_sel = int(np.minimum(nv, 2048).sum())
    pairs = 32768 * 32769 // 2
    sel = 2048 * 2049 // 2 + (32768 - 2048) * 2048
    assert (pairs, n_sel) == (536887296, sel) and sel == 65012736
    f = bench.algorithmic_flops(wl, n_sel)
    assert f["indexer"] == pairs * 64 * 128 * 2 == 8796361457664
    assert f["sparse_mla"] == sel * 128 * (576 + 512) * 2 == 18107867332608
    assert f["step"] == f["indexer"] + f["sparse_mla"]
