"""The chained decode calls keep the stream's order under programmatic
dependent launch.

dsa_fused_decode launches its first kernel (the indexer) with programmatic
dependent launch, so it may be scheduled while the stream's previous kernel
is still running, and that kernel may let dependents start early and write
the call's inputs afterwards. The library's delayed-copy test hook does
exactly that: it lets dependents start at once, sleeps 2 ms and only then
writes the index queries. The call must read the new queries: its selection
and attention must match the oracle on the new values (stale zero queries
would give every score 0 and select the first K positions). The
allocation-free entry point, which launches without programmatic edges, is
held to the same order. (A build whose indexer read its inputs before
waiting also passed here: the early start was not observed on this driver,
so the test guards the ordering contract rather than reproducing a race.)
"""
import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import device as DV
from indexed_sparse_attention_relu_b200 import workloads as W

from gpu_helpers import assert_status_ok, check_attention, check_topk_band

pytestmark = pytest.mark.gpu

DELAY_NS = 2_000_000


def _stale_then_delayed(dw, stream):
    """Zero the index queries, then enqueue the delayed copy of the real ones."""
    real = dw.q_idx.clone()
    dw.q_idx.zero_()
    torch.cuda.synchronize()
    B.dsa_debug_delayed_copy(dw.q_idx, real, DELAY_NS, stream=stream)
    return real


@pytest.mark.parametrize("entry", ["workspace", "noalloc"])
def test_chained_call_reads_inputs_written_after_an_early_trigger(entry):
    wl = W.scaled("c2", B=4, Lmax=3000, lens=(3000, 2100, 1500, 700), T_per_seq=1, K=512)
    dw = DV.to_device(wl)
    out = torch.empty((wl.T, wl.H, wl.dc), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.T, wl.H), dtype=torch.float32, device="cuda")
    idx = torch.full((wl.T, wl.K), -7, dtype=torch.int32, device="cuda")
    nb = B.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, dw.batch, wl.K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()  # an ordinary stream (the legacy default stream has its own rules)
    real = _stale_then_delayed(dw, s)
    if entry == "workspace":
        B.dsa_fused_decode(dw.batch, dw.indexer_in(), dw.mla_in(), wl.K, out, lse, idx, ws, nb, stream=s)
    else:
        B.dsa_fused_decode_noalloc(dw.batch, dw.indexer_in(), dw.mla_in(), wl.K, out, lse, idx, stream=s)
    torch.cuda.synchronize()
    assert_status_ok()
    assert torch.equal(dw.q_idx, real)  # the copy itself landed
    got = idx.cpu().numpy()
    sc = oracle.indexer_scores(wl)
    check_topk_band(got, oracle.topk(sc, wl.n_valid(), wl.K), sc, wl.K)
    # the stale queries would have selected the first K positions of every row
    assert not all(np.array_equal(got[t], np.arange(wl.K)) for t in range(wl.T))
    want_out, want_lse = oracle.sparse_mla(wl, got)
    check_attention(out, lse, want_out, want_lse)
