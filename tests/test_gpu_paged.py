"""GPU parity of paged caches: every cache (index keys, FP8 scales, latent KV
rows) moved into one page pool under a block table, in a seeded random page
order (paged key cache read directly by the fused indexer, section 3 of
"Optimizing Inference for New Model Architectures ...").

Two checks per case:
  * the paged call returns exactly (bit for bit) what the contiguous call on
    the same logical data returns: the kernels read the same rows in the same
    order, only their addresses differ;
  * against the oracle run on the logical cache that ``oracle.unpage`` reads
    back out of the pool (scores within the fp32 bound, indices within the
    tie band, attention within max-abs 1e-2 / rel-L2 5e-3).
Unused table entries are -1, so a kernel that looked up a page a sequence
does not need would set DSA_ERR_DEVICE_INDEX; every case checks the status.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import device as DV
from indexed_sparse_attention_relu_b200 import workloads as W

from gpu_helpers import (assert_status_ok, check_attention, check_scores, check_topk_band, gpu_fused, gpu_mla,
                         gpu_scores, oracle_codes, score_bound)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    B.dsa_read_device_status()
    yield


def _np(t):
    return t.cpu().numpy()


def _same(a, b):
    x = a.view(torch.int16) if a.dtype == torch.bfloat16 else a
    y = b.view(torch.int16) if b.dtype == torch.bfloat16 else b
    return torch.equal(x, y)


def _bf16_unpage(t, table, ps, Lmax):
    bits = oracle.unpage(_np(t.view(torch.int16)).view(np.uint16), table, ps, Lmax)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _logical(pdw):
    """The workload as the oracle sees it: every cache read back out of the
    pool with oracle.unpage. Returns (workload, FP8 codes, FP8 scales); the
    last two are None for BF16 keys."""
    wl = pdw.wl
    table = _np(pdw.batch.block_table)
    ps = pdw.batch.struct.page_size
    kv = _bf16_unpage(pdw.kv, table, ps, wl.Lmax)
    if pdw.k_scale is not None:
        k8 = oracle.unpage(_np(pdw.k_cache), table, ps, wl.Lmax)
        ks = oracle.unpage(_np(pdw.k_scale), table, ps, wl.Lmax)
        return dataclasses.replace(wl, kv=kv), k8, ks
    return dataclasses.replace(wl, k_idx=_bf16_unpage(pdw.k_cache, table, ps, wl.Lmax), kv=kv), None, None


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("page_size", [64, 128, 256])
def test_paged_decode_indexer_matches_contiguous(key_dtype, page_size):
    """One query per sequence (the one-CTA-per-SM decode kernel), ragged
    lengths that end inside a page and inside a 64-row half."""
    wl = W.scaled("c2", B=5, Lmax=1000, lens=(1000, 1, 321, 640, 77), T_per_seq=1, K=128, key_dtype=key_dtype)
    dw = DV.to_device(wl)
    pdw = DV.to_paged(dw, page_size, seed=page_size)
    want = gpu_scores(dw)
    got = gpu_scores(pdw)
    nv = wl.n_valid()
    for t in range(wl.T):
        n = (int(nv[t]) + 127) // 128 * 128
        assert torch.equal(got[t, :n], want[t, :n]), t


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_paged_prefill_indexer_matches_contiguous(key_dtype):
    """Several tokens per sequence (4-token MMA groups) over 64-row pages."""
    wl = W.scaled("c4", B=2, Lmax=700, lens=(700, 333), T_per_seq=150, K=128, key_dtype=key_dtype)
    dw = DV.to_device(wl)
    pdw = DV.to_paged(dw, 64, seed=3)
    want = gpu_scores(dw)
    got = gpu_scores(pdw)
    nv = wl.n_valid()
    for t in range(wl.T):
        n = (int(nv[t]) + 127) // 128 * 128
        assert torch.equal(got[t, :n], want[t, :n]), t


@pytest.mark.parametrize("H", [128, 64])
def test_paged_attention_matches_contiguous(H):
    """Both attention kernels (score/value CTA pairs for 128 heads, one CTA
    per 64-head block otherwise) gather rows through the block table."""
    wl = W.scaled("c2", B=3, Lmax=900, lens=(900, 400, 130), T_per_seq=4, K=300, H=H)
    rng = np.random.default_rng(5)
    nv = wl.n_valid()
    idx = np.full((wl.T, wl.K), -1, np.int32)
    for t in range(wl.T):
        m = min(wl.K - 7, nv[t])
        idx[t, :m] = rng.choice(nv[t], m, replace=False)
        rng.shuffle(idx[t])
    dw = DV.to_device(wl)
    pdw = DV.to_paged(dw, 128, seed=9)
    it = torch.from_numpy(idx).to(dw.q.device)
    o1, l1 = gpu_mla(dw, it)
    o2, l2 = gpu_mla(pdw, it)
    assert _same(o1, o2) and _same(l1, l2)


def test_paged_fused_decode_bf16_matches_oracle():
    """The whole chain on paged caches against the oracle on the unpaged
    logical caches."""
    wl = W.scaled("c2", B=4, Lmax=3000, lens=(3000, 1100, 2048, 77), T_per_seq=1, K=1024)
    dw = DV.to_device(wl)
    pdw = DV.to_paged(dw, 64, seed=11)
    out, lse, idx = gpu_fused(pdw)
    lwl, _, _ = _logical(pdw)
    sc = oracle.indexer_scores(lwl)
    want_idx = oracle.topk(sc, lwl.n_valid(), lwl.K)
    check_topk_band(_np(idx), want_idx, sc, lwl.K)
    want_out, want_lse = oracle.sparse_mla(lwl, _np(idx))
    check_attention(out, lse, want_out, want_lse)
    ref = gpu_fused(dw)
    assert all(_same(a, b) for a, b in zip((out, lse, idx), ref))


def test_paged_fp8_fused_decode_matches_oracle():
    """FP8 index keys: codes and per-key scales both come out of the pool."""
    wl = W.scaled("c3", B=3, Lmax=2500, lens=(2500, 700, 1300), T_per_seq=1, K=512)
    dw = DV.to_device(wl)
    codes, scales = oracle_codes(dw)
    pdw = DV.to_paged(dw, 128, seed=13)
    out, lse, idx = gpu_fused(pdw)
    lwl, k8, ks = _logical(pdw)
    nv = wl.n_valid()
    for b in range(wl.B):  # the pool holds the same codes and scales
        assert np.array_equal(k8[b, :wl.seq_lens[b]], codes[b, :wl.seq_lens[b]])
        assert np.array_equal(ks[b, :wl.seq_lens[b]], scales[b, :wl.seq_lens[b]])
    sc = oracle.indexer_scores(wl, k_codes=k8, k_scales=ks)
    got_sc = _np(gpu_scores(pdw))
    check_scores(got_sc, sc, score_bound(wl, k_codes=k8, k_scales=ks), nv)
    want_idx = oracle.topk(sc, nv, wl.K)
    check_topk_band(_np(idx), want_idx, sc, wl.K)
    want_out, want_lse = oracle.sparse_mla(lwl, _np(idx))
    check_attention(out, lse, want_out, want_lse)


def test_bad_page_id_is_flagged_not_dereferenced():
    """A needed table entry outside the pool: the row reads as pool row 0 and
    the status word reports DSA_ERR_DEVICE_INDEX; the next clean call is
    unaffected."""
    wl = W.scaled("c2", B=2, Lmax=600, lens=(600, 300), T_per_seq=1, K=256)
    dw = DV.to_device(wl)
    pdw = DV.to_paged(dw, 64, seed=17)
    bad = pdw.batch.block_table.clone()
    bad[1, 2] = pdw.batch.struct.num_pages + 5
    bbt = B.Batch(pdw.batch.cu_q, pdw.batch.q_pos, pdw.batch.seq_lens, wl.Lmax, block_table=bad,
                  page_size=64, num_pages=pdw.batch.struct.num_pages)
    sc = torch.empty((wl.T, wl.Lmax), dtype=torch.float32, device=dw.q.device)
    B.dsa_indexer_scores(bbt, pdw.indexer_in(), sc)
    assert B.dsa_read_device_status() == B.DSA_ERR_DEVICE_INDEX
    got = gpu_scores(pdw)
    assert_status_ok()
    assert torch.equal(got[0, :640], gpu_scores(dw)[0, :640])
