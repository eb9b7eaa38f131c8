"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The test lowers the kernels' wait limit to 20 ms and makes the 128-head
attention's score CTA withhold its first "P ready" signal (both are test hooks
of the library). The value CTA's wait for that signal then gives up: the
kernel records DSA_ERR_DEVICE_TIMEOUT in the device status word, every role
leaves its loop, tensor memory is released and the launch completes. Nothing
traps or hangs. A normal call right after must succeed and match the oracle,
which shows that the aborted launch left nothing behind (tensor memory,
copies in flight, barrier state).
"""
import time

import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import device as DV
from indexed_sparse_attention_relu_b200 import workloads as W

from gpu_helpers import check_attention, gpu_mla

pytestmark = pytest.mark.gpu


def _case(T_per_seq, K):
    wl = W.scaled("c2", B=1, Lmax=2100, lens=(2100,), T_per_seq=T_per_seq, K=K)
    rng = np.random.default_rng(5)
    nv = wl.n_valid()
    idx = np.full((wl.T, wl.K), -1, np.int32)
    for t in range(wl.T):
        m = min(wl.K, nv[t])
        idx[t, :m] = rng.choice(nv[t], m, replace=False)
    return wl, idx


@pytest.mark.parametrize("T_per_seq,K", [(1, 512), (8, 2048)])
def test_withheld_signal_times_out_and_next_call_is_clean(T_per_seq, K):
    """(1, 512): one query whose few key tiles split over a cluster of pairs
    (the split merge runs after the timeout too); (8, 2048): more tiles per
    pair than P ring slots, so the score CTA also blocks on the stalled value
    CTA and its own wait runs out."""
    wl, idx_np = _case(T_per_seq, K)
    dw = DV.to_device(wl)
    idx = torch.from_numpy(idx_np).cuda()
    assert B.dsa_read_device_status() == B.DSA_OK
    try:
        B.dsa_debug_set_wait_limit(20_000_000)      # 20 ms
        B.dsa_debug_withhold_signal(True)
        t0 = time.perf_counter()
        gpu_mla(dw, idx, expect_status_ok=False)    # synchronises
        elapsed = time.perf_counter() - t0
        code = B.dsa_read_device_status()
    finally:
        B.dsa_debug_withhold_signal(False)
        B.dsa_debug_set_wait_limit(0)
    assert code == B.DSA_ERR_DEVICE_TIMEOUT, B.status_string(code)
    assert elapsed < 1.0, f"the aborted launch took {elapsed:.3f} s"
    assert B.dsa_read_device_status() == B.DSA_OK   # sticky until read, then clear
    # the next call on the same context is healthy and correct
    out, lse = gpu_mla(dw, idx)
    want_out, want_lse = oracle.sparse_mla(wl, idx_np)
    check_attention(out, lse, want_out, want_lse)
