"""The allocation-free decode entry point, dsa_fused_decode_noalloc.

Some callers cannot give this library device memory at call time: a runtime
or plugin host that owns all device memory through its own pool and passes
extensions no workspace, or a serving path that must never enter the CUDA
allocator. For them the library offers the decode chain with its scratch in
one fixed 32 MiB device array built into libdsa.so. These tests call it
through the C ABI and check it against the workspace-taking entry point
(dsa_fused_decode) on the same inputs, twice in a row, since every call
reuses the same array.
"""
import ctypes

import numpy as np
import pytest
import torch

from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import build as build_mod

MAX_ABS = 1e-2   # attention tolerances used by all parity tests
REL_L2 = 5e-3
SCRATCH = 32 << 20


def test_oversized_call_is_rejected_before_any_work():
    """Runs without a GPU: the size check happens on the host first."""
    build_mod.build()
    lib = B.load()
    fake = 0x10000
    bt = B.dsa_batch(2, 64, 200_000, fake, fake, fake, None, 0)   # 64 * 200000 * 4 B > 32 MiB
    ii = B.dsa_indexer_in(64, 128, fake, fake, B.DSA_KEY_BF16, fake, None, 128)
    mi = B.dsa_mla_in(128, 512, 64, 0.04, fake, fake)
    r = lib.dsa_fused_decode_noalloc(ctypes.byref(bt), ctypes.byref(ii), ctypes.byref(mi), 2048, fake, None, None, None)
    assert r == B.DSA_ERR_WORKSPACE_TOO_SMALL
    assert str(SCRATCH) in B.last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    from indexed_sparse_attention_relu_b200 import device as DV
    from indexed_sparse_attention_relu_b200 import workloads as W

    B.load()
    wl = W.scaled("c2", B=4, Lmax=3000, lens=(3000, 2100, 1500, 700), T_per_seq=2, K=2048)
    dw = DV.to_device(wl, "cuda")
    T, K = wl.T, wl.K
    assert T * wl.Lmax * 4 + T * K * 4 < SCRATCH

    out_ref = torch.empty((T, wl.H, wl.dc), dtype=torch.bfloat16, device="cuda")
    lse_ref = torch.empty((T, wl.H), dtype=torch.float32, device="cuda")
    idx_ref = torch.empty((T, K), dtype=torch.int32, device="cuda")
    nbytes = B.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, dw.batch, K)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    B.dsa_fused_decode(dw.batch, dw.indexer_in(), dw.mla_in(), K, out_ref, lse_ref, idx_ref, ws, nbytes)
    torch.cuda.synchronize()
    ref = out_ref.float().cpu().numpy().astype(np.float64)
    ref_lse = lse_ref.cpu().numpy()

    for call in range(2):
        out = torch.full((T, wl.H, wl.dc), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
        # first call: indices kept in the built-in scratch; second: written to idx_out
        B.dsa_fused_decode_noalloc(dw.batch, dw.indexer_in(), dw.mla_in(), K, out, lse,
                                   idx if call == 1 else None)
        torch.cuda.synchronize()
        assert B.dsa_read_device_status() == B.DSA_OK
        if call == 1:
            assert torch.equal(idx, idx_ref)
        d = out.float().cpu().numpy().astype(np.float64) - ref
        max_abs = float(np.abs(d).max())
        rel = float(np.linalg.norm(d) / np.linalg.norm(ref))
        assert max_abs <= MAX_ABS and rel <= REL_L2, (call, max_abs, rel)
        assert np.allclose(lse.cpu().numpy(), ref_lse, rtol=1e-4, atol=1e-4)


def _noalloc_run(dw, K, with_idx_out):
    wl = dw.wl
    T = wl.T
    out = torch.full((T, wl.H, wl.dc), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, K), -7, dtype=torch.int32, device="cuda") if with_idx_out else None
    B.dsa_fused_decode_noalloc(dw.batch, dw.indexer_in(), dw.mla_in(), K, out, lse, idx)
    torch.cuda.synchronize()
    assert B.dsa_read_device_status() == B.DSA_OK
    return out, lse, idx


@pytest.mark.gpu
def test_noalloc_against_the_oracle_fp8_small_latent():
    """The other branches of the entry point: FP8 index keys (written by the
    library's own cache-write call) and the small-latent attention shape
    (d_c = 64, d_rope = 16, 4 heads), on integer-valued inputs so the selected
    indices are exact; attention checked against the fp64 oracle directly."""
    import oracle
    from gpu_helpers import check_attention
    from indexed_sparse_attention_relu_b200 import device as DV
    from indexed_sparse_attention_relu_b200 import workloads as W

    B.load()
    wl = W.scaled("c5i", B=2, Lmax=700, lens=(700, 300), T_per_seq=3, K=64, key_dtype="fp8", integer=True,
                  HI=4, dI=32, H=4, dc=64, dr=16)
    dw = DV.to_device(wl, "cuda")
    codes, scales = oracle.quantize_keys(wl.k_idx, wl.scale_group)
    _, want_idx, want_out, want_lse = oracle.dsa(wl, rank_in_fp32=True, k_codes=codes, k_scales=scales)
    for call in range(2):
        out, lse, idx = _noalloc_run(dw, wl.K, with_idx_out=True)
        assert np.array_equal(idx.cpu().numpy(), want_idx), call
        check_attention(out, lse, want_out, want_lse)


@pytest.mark.gpu
def test_noalloc_against_the_oracle_decode_shape():
    """128 heads, 576/512 latent rows, BF16 keys: indices within the tie band of
    the oracle's selection and attention against the oracle on those indices."""
    import oracle
    from gpu_helpers import check_attention, check_topk_band
    from indexed_sparse_attention_relu_b200 import device as DV
    from indexed_sparse_attention_relu_b200 import workloads as W

    B.load()
    wl = W.scaled("c2", B=3, Lmax=2600, lens=(2600, 2049, 900), T_per_seq=1, K=2048)
    dw = DV.to_device(wl, "cuda")
    out, lse, idx = _noalloc_run(dw, wl.K, with_idx_out=True)
    sc = oracle.indexer_scores(wl)
    got_idx = idx.cpu().numpy()
    check_topk_band(got_idx, oracle.topk(sc, wl.n_valid(), wl.K), sc, wl.K)
    want_out, want_lse = oracle.sparse_mla(wl, got_idx)
    check_attention(out, lse, want_out, want_lse)


@pytest.mark.gpu
def test_noalloc_scratch_filled_to_its_last_byte():
    """num_q * max_seq_len * 4 + num_q * k * 4 equals the 32 MiB limit exactly:
    the last query's score row and the index tail (no idx_out) reach the end of
    the built-in array. Checked against the workspace entry point."""
    from indexed_sparse_attention_relu_b200 import device as DV
    from indexed_sparse_attention_relu_b200 import workloads as W

    B.load()
    T, K = 64, 2048
    Lmax = (SCRATCH - T * K * 4) // (T * 4)
    assert T * Lmax * 4 % 256 == 0 and T * Lmax * 4 + T * K * 4 == SCRATCH
    wl = W.scaled("c2", B=1, Lmax=Lmax, lens=(2500,), T_per_seq=T, K=K)
    dw = DV.to_device(wl, "cuda")
    nbytes = B.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, dw.batch, K)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out_ref = torch.empty((T, wl.H, wl.dc), dtype=torch.bfloat16, device="cuda")
    idx_ref = torch.empty((T, K), dtype=torch.int32, device="cuda")
    B.dsa_fused_decode(dw.batch, dw.indexer_in(), dw.mla_in(), K, out_ref, None, idx_ref, ws, nbytes)
    torch.cuda.synchronize()
    ref = out_ref.float().cpu().numpy().astype(np.float64)
    for call in range(2):
        out, _, _ = _noalloc_run(dw, K, with_idx_out=False)
        d = out.float().cpu().numpy().astype(np.float64) - ref
        assert float(np.abs(d).max()) <= MAX_ABS and float(np.linalg.norm(d) / np.linalg.norm(ref)) <= REL_L2, call
    # one byte more is rejected on the host
    bt = B.dsa_batch(1, T, Lmax + 1, 0x10000, 0x10000, 0x10000, None, 0)
    r = B.load().dsa_fused_decode_noalloc(ctypes.byref(bt), ctypes.byref(dw.indexer_in()), ctypes.byref(dw.mla_in()),
                                          K, 0x10000, None, None, None)
    assert r == B.DSA_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.gpu
def test_noalloc_paged_caches_and_fp8_kv():
    """Paged caches (64-row pages under one block table) with an FP8 latent KV
    cache: the allocation-free call matches the workspace entry point on the
    same inputs (indices identical; the attention runs unsplit here)."""
    from indexed_sparse_attention_relu_b200 import device as DV
    from indexed_sparse_attention_relu_b200 import workloads as W

    B.load()
    wl = W.scaled("c2", B=3, Lmax=2600, lens=(2600, 2049, 900), T_per_seq=1, K=1024)
    dw = DV.to_paged(DV.with_fp8_kv(DV.to_device(wl, "cuda")), 64, seed=5)
    T, K = wl.T, wl.K
    nbytes = B.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, dw.batch, K)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out_ref = torch.empty((T, wl.H, wl.dc), dtype=torch.bfloat16, device="cuda")
    idx_ref = torch.empty((T, K), dtype=torch.int32, device="cuda")
    B.dsa_fused_decode(dw.batch, dw.indexer_in(), dw.mla_in(), K, out_ref, None, idx_ref, ws, nbytes)
    torch.cuda.synchronize()
    ref = out_ref.float().cpu().numpy().astype(np.float64)
    for call in range(2):
        out, _, idx = _noalloc_run(dw, K, with_idx_out=True)
        assert torch.equal(idx, idx_ref), call
        d = out.float().cpu().numpy().astype(np.float64) - ref
        assert float(np.abs(d).max()) <= MAX_ABS and float(np.linalg.norm(d) / np.linalg.norm(ref)) <= REL_L2, call
