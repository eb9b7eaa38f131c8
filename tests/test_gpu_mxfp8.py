"""GPU parity of MXFP8 index queries and keys (Index Q/K Uses MXFP8, section
4.2 of "Inference Adaptation and Performance Optimization for New Large
Language Model Architectures": 32 elements per scale factor).

  * dsa_quantize_mxfp8 is bit-exact against oracle.mx_quantize (codes and
    E8M0 scale bytes);
  * the indexer on MXFP8 inputs matches the oracle run on the dequantised
    queries and keys: those values are exact in bf16, so the bf16 fp32-sum
    bound applies unchanged; integer inputs are bit-exact;
  * both kernels (one CTA per SM for decode, token groups for prefill), the
    scale bytes staged with the codes or read from global memory, paged
    caches, and the fused decode chain.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import device as DV
from indexed_sparse_attention_relu_b200 import workloads as W

from gpu_helpers import check_attention, check_scores, check_topk_band, gpu_fused, score_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    B.dsa_read_device_status()
    yield


def _np(t):
    return t.cpu().numpy()


def _mx_view(wl):
    """The workload as MXFP8 leaves it: queries and keys replaced by the
    oracle's dequantised MXFP8 values (exact in fp32)."""
    qc, qs = oracle.mx_quantize(wl.q_idx)
    kc, ks = oracle.mx_quantize(wl.k_idx)
    return dataclasses.replace(wl, q_idx=oracle.mx_dequantize(qc, qs).astype(np.float32),
                               k_idx=oracle.mx_dequantize(kc, ks).astype(np.float32)), (qc, qs, kc, ks)


def _scores(dw):
    wl = dw.wl
    sc = torch.full((wl.T, wl.Lmax), float("nan"), dtype=torch.float32, device=dw.q.device)
    nb = B.dsa_workspace_size(B.DSA_OP_INDEXER_SCORES, dw.batch, wl.K, wl.HI, wl.dI)
    ws = torch.empty(nb, dtype=torch.uint8, device=dw.q.device)
    B.dsa_indexer_scores(dw.batch, dw.indexer_in(), sc, None, ws, nb)
    assert B.dsa_read_device_status() == B.DSA_OK
    return _np(sc)


@pytest.mark.parametrize("dim", [128, 32])
def test_quantize_mxfp8_bit_exact(dim):
    rng = np.random.default_rng(dim)
    x = rng.standard_normal((300, dim)).astype(np.float32) * np.exp(rng.uniform(-8, 8, (300, 1))).astype(np.float32)
    x[4] = 0.0
    x[9, :32] = 448.0 * 2.0 ** -3     # absmax exactly on a power-of-two boundary
    x = W.bf16_round(x)
    dev = torch.device("cuda", 0)
    xt = DV.bf16_tensor(x, dev)
    codes = torch.empty(x.shape, dtype=torch.uint8, device=dev)
    sb = torch.empty((300, dim // 32), dtype=torch.uint8, device=dev)
    B.dsa_quantize_mxfp8(xt, codes, sb)
    want_c, want_s = oracle.mx_quantize(x)
    assert np.array_equal(_np(sb), want_s)
    assert np.array_equal(_np(codes), want_c)


@pytest.mark.parametrize("HI,dI", [(64, 128), (4, 32)])
def test_mxfp8_decode_integer_exact(HI, dI):
    """Integer values in [-2, 2]: MXFP8 holds them exactly, every score is an
    exact integer, so the kernel must match the oracle bit for bit."""
    wl = W.scaled("c5i", B=4, Lmax=700, lens=(700, 129, 1, 513), T_per_seq=1, K=64, HI=HI, dI=dI,
                  key_dtype="bf16", integer=True)
    mwl, _ = _mx_view(wl)
    assert np.array_equal(mwl.k_idx, wl.k_idx) and np.array_equal(mwl.q_idx, wl.q_idx)
    dw = DV.with_mxfp8_index(DV.to_device(wl))
    got = _scores(dw)
    want = oracle.indexer_scores(mwl)
    nv = wl.n_valid()
    for t in range(wl.T):
        assert np.array_equal(got[t, :nv[t]], want[t, :nv[t]].astype(np.float32)), t


@pytest.mark.parametrize("Lmax", [2000, 2001])
def test_mxfp8_decode_matches_oracle(Lmax):
    """Normal values, ragged lengths; L_max a multiple of 4 stages the scale
    bytes with the codes, otherwise the converters read them from memory."""
    wl = W.scaled("c2", B=5, Lmax=Lmax, lens=(Lmax, 1, 700, 1999, 130), T_per_seq=1, K=256, key_dtype="bf16")
    mwl, (qc, qs, kc, ks) = _mx_view(wl)
    dw = DV.with_mxfp8_index(DV.to_device(wl))
    assert np.array_equal(_np(dw.k_cache), kc) and np.array_equal(_np(dw.k_mx), ks)
    got = _scores(dw)
    check_scores(got, oracle.indexer_scores(mwl), score_bound(mwl), wl.n_valid())


def test_mxfp8_prefill_groups_matches_oracle():
    """Several tokens per sequence: the 4-token group kernel."""
    wl = W.scaled("c4", B=2, Lmax=700, lens=(700, 333), T_per_seq=150, K=128, key_dtype="bf16")
    mwl, _ = _mx_view(wl)
    dw = DV.with_mxfp8_index(DV.to_device(wl))
    got = _scores(dw)
    check_scores(got, oracle.indexer_scores(mwl), score_bound(mwl), wl.n_valid())


@pytest.mark.parametrize("T_per_seq", [1, 150])
def test_mxfp8_paged_matches_contiguous(T_per_seq):
    wl = W.scaled("c4", B=2, Lmax=700, lens=(700, 333), T_per_seq=T_per_seq, K=128, key_dtype="bf16")
    dw = DV.with_mxfp8_index(DV.to_device(wl))
    pdw = DV.to_paged(dw, 64, seed=31)
    a, b = _scores(dw), _scores(pdw)
    nv = wl.n_valid()
    for t in range(wl.T):
        n = (int(nv[t]) + 127) // 128 * 128
        assert np.array_equal(a[t, :n], b[t, :n]), t


def test_mxfp8_fused_decode():
    wl = W.scaled("c2", B=4, Lmax=3000, lens=(3000, 1100, 2048, 77), T_per_seq=1, K=1024, key_dtype="bf16")
    mwl, _ = _mx_view(wl)
    dw = DV.with_mxfp8_index(DV.to_device(wl))
    out, lse, idx = gpu_fused(dw)
    sc = oracle.indexer_scores(mwl)
    check_topk_band(_np(idx), oracle.topk(sc, wl.n_valid(), wl.K), sc, wl.K)
    want_out, want_lse = oracle.sparse_mla(wl, _np(idx))
    check_attention(out, lse, want_out, want_lse)
