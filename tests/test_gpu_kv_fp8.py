"""GPU parity of the FP8 latent-KV cache (block-wise FP8 KV cache: section 4
of "Optimizing Inference for New Model Architectures ..."; Tiered
Quantization table of "Day-0 Inference Adaptation ...").

  * the cache write (dsa_quantize_kv) is bit-exact against the oracle's
    codes, scales and rope dims, packed in the row layout the header states;
  * attention over FP8 rows matches the oracle run on the rows dequantised in
    fp64 (max-abs 1e-2, rel-L2 5e-3, lse 1e-3): the kernel widens each
    element to bf16 (one rounding of fl32(code * scale)), inside that bound;
  * paged FP8 rows give bit-identical results to contiguous ones.
"""
import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import device as DV
from indexed_sparse_attention_relu_b200 import workloads as W

from gpu_helpers import check_attention, check_topk_band, gpu_fused, gpu_mla, oracle_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    B.dsa_read_device_status()
    yield


def _np(t):
    return t.cpu().numpy()


def _pack(codes, scales, rope):
    """Rows in the header's layout: codes | rope bf16 | fp32 scales | zeros."""
    n = codes.shape[0]
    dc, dr, nt = codes.shape[1], rope.shape[1], scales.shape[1]
    row = B.dsa_kv_fp8_row_bytes(dc, dr)
    out = np.zeros((n, row), np.uint8)
    out[:, :dc] = codes
    out[:, dc:dc + 2 * dr] = W.bf16_bits(rope).view(np.uint8).reshape(n, 2 * dr)
    out[:, dc + 2 * dr:dc + 2 * dr + 4 * nt] = np.ascontiguousarray(scales, np.float32).view(np.uint8).reshape(n, 4 * nt)
    return out


def _kv64(wl):
    codes, scales, rope = oracle.quantize_kv(wl.kv, dc=wl.dc)
    return oracle.dequantize_kv(codes, scales, rope)


@pytest.mark.parametrize("name", ["c2", "c1"])
def test_quantize_kv_bit_exact(name):
    wl = W.scaled(name, B=2, Lmax=300, lens=(300, 123), T_per_seq=1, K=8) if name == "c2" else W.make("c1")
    rows = wl.kv.reshape(-1, wl.D)
    rng = np.random.default_rng(4)
    rows = rows.copy()
    rows[3] = 0.0                                         # all-zero row: scales 0, codes 0
    rows[5, :wl.dc] *= 1e-30                              # tiny values: subnormal codes / scales
    rows = W.bf16_round(rows)
    dev = torch.device("cuda", 0)
    src = DV.bf16_tensor(rows, dev)
    got = torch.full((rows.shape[0], B.dsa_kv_fp8_row_bytes(wl.dc, wl.dr)), 0xAB, dtype=torch.uint8, device=dev)
    B.dsa_quantize_kv(src, wl.dc, got)
    want = _pack(*oracle.quantize_kv(rows, dc=wl.dc))
    assert np.array_equal(_np(got), want)


@pytest.mark.parametrize("T_per_seq,H", [(1, 128), (16, 128), (1, 64), (40, 64)])
def test_mla_fp8_kv_matches_oracle(T_per_seq, H):
    """128 heads run as two 64-head blocks; 1 query per sequence splits the
    keys (merge through the workspace), 16/40 do not."""
    wl = W.scaled("c2", B=2, Lmax=900, lens=(900, 400), T_per_seq=T_per_seq, K=300, H=H)
    rng = np.random.default_rng(T_per_seq + H)
    nv = wl.n_valid()
    idx = np.full((wl.T, wl.K), -1, np.int32)
    for t in range(wl.T):
        m = min(wl.K - 7, nv[t])
        idx[t, :m] = rng.choice(nv[t], m, replace=False)
        rng.shuffle(idx[t])
    dw = DV.with_fp8_kv(DV.to_device(wl))
    out, lse = gpu_mla(dw, torch.from_numpy(idx).to(dw.q.device))
    want_out, want_lse = oracle.sparse_mla(wl, idx, kv=_kv64(wl))
    check_attention(out, lse, want_out, want_lse)


def test_mla_fp8_kv_small_latent():
    wl = W.make("c1")
    sc = oracle.indexer_scores(wl)
    idx = oracle.topk(sc, wl.n_valid(), wl.K)
    dw = DV.with_fp8_kv(DV.to_device(wl))
    out, lse = gpu_mla(dw, torch.from_numpy(idx).to(dw.q.device))
    want_out, want_lse = oracle.sparse_mla(wl, idx, kv=_kv64(wl))
    check_attention(out, lse, want_out, want_lse)


def test_mla_fp8_kv_single_key_is_the_widened_row():
    """K = 1: out is the selected row's latent part as the kernel widens it,
    bf16(fl32(decode(code) * scale)), exactly."""
    wl = W.scaled("c2", B=1, Lmax=300, lens=(300,), T_per_seq=3, K=1, H=64)
    idx = np.array([[17], [250], [0]], np.int32)
    dw = DV.with_fp8_kv(DV.to_device(wl))
    out, _ = gpu_mla(dw, torch.from_numpy(idx).to(dw.q.device))
    codes, scales, _ = oracle.quantize_kv(wl.kv, dc=wl.dc)
    for r in range(3):
        s = idx[r, 0]
        x = (oracle.e4m3_decode(codes[0, s]).astype(np.float32) * np.repeat(scales[0, s], 128)).astype(np.float32)
        want = W.bf16_round(x)
        got = out[r].float().cpu().numpy()
        assert np.array_equal(got, np.broadcast_to(want, got.shape)), r


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_fused_decode_fp8_kv(key_dtype):
    wl = W.scaled("c3", B=4, Lmax=3000, lens=(3000, 1100, 2048, 77), T_per_seq=1, K=1024, key_dtype=key_dtype)
    dw = DV.with_fp8_kv(DV.to_device(wl))
    out, lse, idx = gpu_fused(dw)
    kw = {}
    if key_dtype == "fp8":
        codes, scales = oracle_codes(dw)
        kw = dict(k_codes=codes, k_scales=scales)
    sc = oracle.indexer_scores(wl, **kw)
    check_topk_band(_np(idx), oracle.topk(sc, wl.n_valid(), wl.K), sc, wl.K)
    want_out, want_lse = oracle.sparse_mla(wl, _np(idx), kv=_kv64(wl))
    check_attention(out, lse, want_out, want_lse)


def test_paged_fp8_kv_matches_contiguous():
    wl = W.scaled("c2", B=3, Lmax=900, lens=(900, 400, 130), T_per_seq=4, K=300)
    rng = np.random.default_rng(8)
    nv = wl.n_valid()
    idx = np.full((wl.T, wl.K), -1, np.int32)
    for t in range(wl.T):
        m = min(wl.K - 7, nv[t])
        idx[t, :m] = rng.choice(nv[t], m, replace=False)
    dw = DV.with_fp8_kv(DV.to_device(wl))
    pdw = DV.to_paged(dw, 64, seed=21)
    it = torch.from_numpy(idx).to(dw.q.device)
    o1, l1 = gpu_mla(dw, it)
    o2, l2 = gpu_mla(pdw, it)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)
