"""GPU checks of the DSA_DEBUG build (libdsa_debug.so).

  * small cases of every tensor-core kernel (decode indexer, 4-token group
    indexer, 128-head CTA pairs, 64-head kernel, FP8 keys) run clean: the
    shared-memory canaries stay intact (status DSA_OK) and the results match
    the oracle as in the release build;
  * an index outside its sequence, handed to dsa_sparse_mla_attn, is caught
    on the host before anything is launched (DSA_ERR_INVALID_ARGUMENT naming
    the row and position), where the release build skips it on the device.
"""
import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import build as build_mod
from indexed_sparse_attention_relu_b200 import device as DV
from indexed_sparse_attention_relu_b200 import workloads as W

from gpu_helpers import check_attention, check_scores, check_topk_band, gpu_fused, gpu_scores, oracle_codes, score_bound

pytestmark = pytest.mark.gpu


@pytest.fixture
def debug_lib():
    """Routes the binding to libdsa_debug.so for one test, then back."""
    release = B.LIB_PATH
    B.dsa_read_device_status()
    B._lib = None
    B.LIB_PATH = build_mod.build(debug=True)
    B.load()
    B.dsa_read_device_status()
    yield
    B._lib = None
    B.LIB_PATH = release
    B.load()


def _np(t):
    return t.cpu().numpy()


def test_debug_c1_fused_decode_is_bit_exact_and_clean(debug_lib):
    wl = W.make("c1")
    dw = DV.to_device(wl)
    out, lse, idx = gpu_fused(dw)          # asserts the status word is clean
    sc, want_idx, want_out, want_lse = oracle.dsa(wl, rank_in_fp32=True)
    assert np.array_equal(_np(idx), want_idx)
    check_attention(out, lse, want_out, want_lse)


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_debug_ragged_decode_clean(debug_lib, key_dtype):
    wl = W.scaled("c3", B=4, Lmax=3000, lens=(3000, 1100, 2048, 77), T_per_seq=1, K=1024, key_dtype=key_dtype)
    dw = DV.to_device(wl)
    out, lse, idx = gpu_fused(dw)
    kw = {}
    if key_dtype == "fp8":
        codes, scales = oracle_codes(dw)
        kw = dict(k_codes=codes, k_scales=scales)
    sc = oracle.indexer_scores(wl, **kw)
    check_topk_band(_np(idx), oracle.topk(sc, wl.n_valid(), wl.K), sc, wl.K)
    want_out, want_lse = oracle.sparse_mla(wl, _np(idx))
    check_attention(out, lse, want_out, want_lse)


def test_debug_prefill_groups_and_64_heads_clean(debug_lib):
    wl = W.scaled("c4", B=2, Lmax=700, lens=(700, 333), T_per_seq=40, K=128, H=64)
    dw = DV.to_device(wl)
    got = _np(gpu_scores(dw))
    check_scores(got, oracle.indexer_scores(wl), score_bound(wl), wl.n_valid())
    out, lse, idx = gpu_fused(dw)
    want_out, want_lse = oracle.sparse_mla(wl, _np(idx))
    check_attention(out, lse, want_out, want_lse)


def test_debug_bad_index_is_caught_on_the_host(debug_lib):
    wl = W.scaled("c2", B=2, Lmax=600, lens=(600, 300), T_per_seq=2, K=128)
    dw = DV.to_device(wl)
    idx = np.tile(np.arange(128, dtype=np.int32), (wl.T, 1))
    idx[3, 17] = 450                       # sequence 1 holds 300 rows
    it = torch.from_numpy(idx).cuda()
    out = torch.empty((wl.T, wl.H, wl.dc), dtype=torch.bfloat16, device="cuda")
    nb = B.dsa_workspace_size(B.DSA_OP_SPARSE_MLA, dw.batch, wl.K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.DsaError) as e:
        B.dsa_sparse_mla_attn(dw.batch, dw.mla_in(), it, wl.K, out, None, ws, nb)
    assert e.value.status == B.DSA_ERR_INVALID_ARGUMENT
    assert "idx[3][17] = 450" in str(e.value)
    assert B.dsa_read_device_status() == B.DSA_OK   # nothing ran
