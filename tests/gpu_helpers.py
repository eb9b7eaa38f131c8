"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare with the oracle under the acceptance rules of the DSA hot path.

Rules (written out in the tests that use them):
  * integer-valued workloads: indexer scores and Top-K indices bit-exact;
  * otherwise a score may differ from the fp64 oracle by at most the fp32
    accumulation bound of its two sums (derived below), and an index-set
    difference is allowed only among positions whose oracle score lies
    within 1e-3 relative of the K-th oracle score;
  * attention outputs: max-abs <= 1e-2 and relative-L2 <= 5e-3 against the
    oracle run on the same indices.
"""
import numpy as np
import torch

import oracle
from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import device as DV

U32 = 2.0 ** -24  # fp32 unit roundoff

MAX_ABS = 1e-2
REL_L2 = 5e-3
TIE_BAND = 1e-3


def gpu_scores(dw, ld=None):
    wl = dw.wl
    ld = ld or wl.Lmax
    scores = torch.full((wl.T, ld), float("nan"), dtype=torch.float32, device=dw.q.device)
    B.dsa_indexer_scores(dw.batch, dw.indexer_in(), scores, ld)
    assert_status_ok()
    return scores


def gpu_topk(dw, scores, K=None):
    wl = dw.wl
    K = K or wl.K
    idx = torch.full((wl.T, K), -7, dtype=torch.int32, device=scores.device)
    B.dsa_topk(dw.batch, scores, K, idx)
    assert_status_ok()
    return idx


def assert_status_ok():
    """Synchronises and checks that no kernel recorded a device-side error
    (an out-of-range index or a bounded wait that gave up)."""
    code = B.dsa_read_device_status()
    assert code == B.DSA_OK, f"device status {code}: {B.status_string(code)}"


def gpu_mla(dw, idx, K=None, expect_status_ok=True):
    wl = dw.wl
    K = K or idx.shape[1]
    out = torch.empty((wl.T, wl.H, wl.dc), dtype=torch.bfloat16, device=dw.q.device)
    lse = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dw.q.device)
    nbytes = B.dsa_workspace_size(B.DSA_OP_SPARSE_MLA, dw.batch, K)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dw.q.device)
    B.dsa_sparse_mla_attn(dw.batch, dw.mla_in(), idx, K, out, lse, ws, nbytes)
    torch.cuda.synchronize()
    if expect_status_ok:
        assert_status_ok()
    return out, lse


def gpu_fused(dw, K=None):
    wl = dw.wl
    K = K or wl.K
    dev = dw.q.device
    out = torch.empty((wl.T, wl.H, wl.dc), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dev)
    idx = torch.full((wl.T, K), -7, dtype=torch.int32, device=dev)
    nbytes = B.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, dw.batch, K)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    B.dsa_fused_decode(dw.batch, dw.indexer_in(), dw.mla_in(), K, out, lse, idx, ws, nbytes)
    assert_status_ok()
    return out, lse, idx


def score_bound(wl, rows=None, k_codes=None, k_scales=None):
    """Per-entry bound on |fp32 kernel score - exact score|.

    The kernel forms each head's dot product with fp32 accumulation of exact
    bf16 x bf16 products (d_I terms), then sum_j w_j relu(.) in fp32 (H_I
    terms) and, for FP8 keys, one multiplication by the key scale. With
    n-term fp32 sums the error is at most n * u * sum|terms| (first order), so
        |err| <= (d_I + H_I + 2) * u * sum_j |w_j| * sum_d |q_jd k_sd| * s_k
    with s_k = 1 for bf16 keys; computed here in fp64 (numpy)."""
    rows = np.arange(wl.T) if rows is None else np.asarray(rows)
    b = wl.seq_of_token()
    out = np.zeros((len(rows), wl.Lmax))
    for r, t in enumerate(rows):
        if k_codes is not None:
            kk = oracle.e4m3_decode(k_codes[b[t]]) * np.abs(k_scales[b[t]].astype(np.float64)).repeat(
                wl.dI // k_scales.shape[-1], -1)
        else:
            kk = wl.k_idx[b[t]].astype(np.float64)
        absdot = np.abs(wl.q_idx[t].astype(np.float64)) @ np.abs(kk).T      # [HI, L]
        out[r] = (wl.dI + wl.HI + 2) * U32 * (np.abs(wl.w[t].astype(np.float64)) @ absdot)
    return out


def check_scores(got, want, bound, n_valid):
    """got/want [rows, L]; masked entries are -inf on both sides."""
    for r in range(got.shape[0]):
        nv = int(n_valid[r])
        g, w = got[r, :nv], want[r, :nv]
        assert np.all(np.isfinite(g)), f"row {r}: non-finite score"
        err = np.abs(g - w)
        bad = err > bound[r, :nv] + 1e-30
        assert not bad.any(), f"row {r}: {bad.sum()} scores outside the fp32 bound, max err {err.max()}"
        tail = got[r, nv:(nv + 127) // 128 * 128]
        assert np.all(tail == -np.inf), f"row {r}: masked tail not -inf"


def check_topk_band(got_idx, want_idx, oracle_scores, K):
    """Index sets may differ only among positions whose oracle score is within
    TIE_BAND relative of the K-th oracle score; both must be valid selections."""
    for r in range(got_idx.shape[0]):
        g = got_idx[r]
        w = want_idx[r]
        gs = set(int(x) for x in g if x >= 0)
        ws = set(int(x) for x in w if x >= 0)
        assert len(gs) == len(ws), f"row {r}: {len(gs)} vs {len(ws)} selected"
        assert list(g[:len(gs)]) == sorted(gs), f"row {r}: not ascending"
        assert np.all(g[len(gs):] == -1)
        if gs == ws:
            continue
        sc = oracle_scores[r]
        kth = np.sort(sc[np.isfinite(sc)])[::-1][min(K, np.isfinite(sc).sum()) - 1]
        for p in gs ^ ws:
            assert abs(sc[p] - kth) <= TIE_BAND * abs(kth), \
                f"row {r}: position {p} (score {sc[p]}) differs outside the tie band of the K-th score {kth}"


def check_attention(out, lse, want_out, want_lse):
    o = out.float().cpu().numpy().astype(np.float64)
    d = o - want_out
    max_abs = np.abs(d).max() if d.size else 0.0
    rel = np.linalg.norm(d) / max(np.linalg.norm(want_out), 1e-30)
    assert max_abs <= MAX_ABS, f"max-abs {max_abs}"
    assert rel <= REL_L2, f"rel-L2 {rel}"
    if lse is not None:
        l = lse.cpu().numpy().astype(np.float64)
        fin = np.isfinite(want_lse)
        assert np.array_equal(np.isfinite(l), fin)
        assert np.abs(l[fin] - want_lse[fin]).max(initial=0.0) <= 1e-3 * max(1.0, np.abs(want_lse[fin]).max(initial=0.0))
    return max_abs, rel


def oracle_codes(dw):
    """The oracle's own FP8 cache write of the workload's keys (and a check
    that the device wrote exactly the same codes and scales)."""
    wl = dw.wl
    codes, scales = oracle.quantize_keys(wl.k_idx, wl.scale_group)
    assert np.array_equal(dw.k_cache.cpu().numpy(), codes), "device FP8 codes differ from the oracle's"
    assert np.array_equal(dw.k_scale.cpu().numpy(), scales), "device FP8 scales differ from the oracle's"
    return codes, scales
