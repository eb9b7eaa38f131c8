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
