"""The C-ABI library loads, exports every symbol include/dsa.h declares, and
rejects bad arguments with a status before anything is enqueued.

These run without a GPU: every call below fails validation, which happens on
the host before any CUDA call, so fake (never dereferenced) pointers are fine.
"""
import ctypes
import os
import re

import pytest

from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(B.EXPORTED) == names


def test_status_strings(lib):
    for s in range(9):
        assert B.status_string(s)
    assert lib.dsa_version().decode().startswith("dsa-b200")


FAKE = 0x10000  # 16-byte aligned, never dereferenced
MIS = 0x10004   # misaligned


def _batch(**kw):
    d = dict(batch=2, num_q=2, max_seq_len=256, cu_q=FAKE, q_pos=FAKE, seq_lens=FAKE, block_table=None, page_size=0)
    d.update(kw)
    return B.dsa_batch(**d)


def _idx_in(**kw):
    d = dict(n_heads=64, head_dim=128, q=FAKE, w=FAKE, key_dtype=B.DSA_KEY_BF16, k_cache=FAKE, k_scale=None,
             scale_group=128)
    d.update(kw)
    return B.dsa_indexer_in(**d)


def _mla_in(**kw):
    d = dict(n_heads=128, d_latent=512, d_rope=64, softmax_scale=0.04, q=FAKE, kv=FAKE)
    d.update(kw)
    return B.dsa_mla_in(**d)


def _scores(lib, batch, inp, scores=FAKE, ld=256):
    return lib.dsa_indexer_scores(ctypes.byref(batch), ctypes.byref(inp), scores, ld, None, 0, None)


def test_indexer_validation(lib):
    assert lib.dsa_indexer_scores(None, ctypes.byref(_idx_in()), FAKE, 256, None, 0, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(batch=0), _idx_in()) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(cu_q=None), _idx_in()) == B.DSA_ERR_INVALID_ARGUMENT
    # paged caches: page_size a positive multiple of 64, a positive page count,
    # a pool below 2^31 rows, an aligned table; no paging fields without a table
    assert _scores(lib, _batch(block_table=FAKE), _idx_in()) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert _scores(lib, _batch(block_table=FAKE, page_size=96, num_pages=4), _idx_in()) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert _scores(lib, _batch(block_table=FAKE, page_size=64, num_pages=0), _idx_in()) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(block_table=FAKE, page_size=1 << 16, num_pages=1 << 15), _idx_in()) == \
        B.DSA_ERR_UNSUPPORTED_SHAPE
    assert _scores(lib, _batch(block_table=FAKE + 2, page_size=64, num_pages=8), _idx_in()) == B.DSA_ERR_MISALIGNED
    assert _scores(lib, _batch(page_size=64), _idx_in()) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(num_pages=3), _idx_in()) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(block_table=FAKE, page_size=128, num_pages=8, num_q=0), _idx_in()) == B.DSA_OK
    assert _scores(lib, _batch(), _idx_in(n_heads=32)) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert _scores(lib, _batch(), _idx_in(head_dim=96)) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert _scores(lib, _batch(), _idx_in(q=MIS)) == B.DSA_ERR_MISALIGNED
    assert _scores(lib, _batch(), _idx_in(key_dtype=7)) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(), _idx_in(key_dtype=B.DSA_KEY_FP8_E4M3)) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(), _idx_in(key_dtype=B.DSA_KEY_FP8_E4M3, k_scale=FAKE, scale_group=32)) == \
        B.DSA_ERR_UNSUPPORTED_SHAPE
    # MXFP8: both scale arrays, groups of 32, and a workspace for the widened queries
    mx = dict(key_dtype=B.DSA_KEY_MXFP8, scale_group=32, q_scale_e8m0=FAKE, k_scale_e8m0=FAKE)
    assert _scores(lib, _batch(), _idx_in(**dict(mx, k_scale_e8m0=None))) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(), _idx_in(**dict(mx, scale_group=128))) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert _scores(lib, _batch(), _idx_in(**dict(mx, q_scale_e8m0=MIS))) == B.DSA_ERR_MISALIGNED
    assert _scores(lib, _batch(), _idx_in(**mx)) == B.DSA_ERR_WORKSPACE_TOO_SMALL
    assert lib.dsa_quantize_mxfp8(FAKE, 4, 48, FAKE, FAKE, None) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert lib.dsa_quantize_mxfp8(FAKE, 4, 64, MIS, FAKE, None) == B.DSA_ERR_MISALIGNED
    assert lib.dsa_fused_decode_noalloc(ctypes.byref(_batch()), ctypes.byref(_idx_in(**mx)), ctypes.byref(_mla_in()),
                                        16, FAKE, None, None, None) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert _scores(lib, _batch(), _idx_in(), scores=None) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(), _idx_in(), ld=100) == B.DSA_ERR_INVALID_ARGUMENT
    assert _scores(lib, _batch(batch=70000, max_seq_len=40000), _idx_in()) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert "shape" in B.last_error() or "2^31" in B.last_error()
    # an empty batch is a no-op
    assert _scores(lib, _batch(num_q=0), _idx_in()) == B.DSA_OK


def test_topk_validation(lib):
    b = _batch()
    assert lib.dsa_topk(ctypes.byref(b), None, 256, 16, FAKE, None, 0, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_topk(ctypes.byref(b), FAKE, 256, 0, FAKE, None, 0, None) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert lib.dsa_topk(ctypes.byref(b), FAKE, 256, 4096, FAKE, None, 0, None) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert lib.dsa_topk(ctypes.byref(b), FAKE, 255, 16, FAKE, None, 0, None) == B.DSA_ERR_INVALID_ARGUMENT


def test_mla_validation(lib):
    b = _batch()

    def call(inp, idx=FAKE, k=64, out=FAKE, ws=None, ws_bytes=0, batch=b):
        return lib.dsa_sparse_mla_attn(ctypes.byref(batch), ctypes.byref(inp), idx, k, out, None, ws, ws_bytes, None)

    assert call(_mla_in(d_latent=256)) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert call(_mla_in(n_heads=96)) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert call(_mla_in(n_heads=0)) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert call(_mla_in(kv=MIS)) == B.DSA_ERR_MISALIGNED
    assert call(_mla_in(softmax_scale=float("nan"))) == B.DSA_ERR_INVALID_ARGUMENT
    assert call(_mla_in(), idx=None) == B.DSA_ERR_INVALID_ARGUMENT
    assert call(_mla_in(), out=MIS) == B.DSA_ERR_MISALIGNED
    assert call(_mla_in(), k=0) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert call(_mla_in(), k=4096) == B.DSA_ERR_UNSUPPORTED_SHAPE
    # key-split partials merge through the workspace; a tiny batch splits its keys
    assert lib.dsa_workspace_size(B.DSA_OP_SPARSE_MLA, ctypes.byref(b), 2048, 64, 128) > 0


def test_fused_and_quant_validation(lib):
    b = _batch()
    r = lib.dsa_fused_decode(ctypes.byref(b), ctypes.byref(_idx_in()), ctypes.byref(_mla_in()), 2048, FAKE, None,
                             None, None, 0, None, None)
    assert r == B.DSA_ERR_WORKSPACE_TOO_SMALL
    need = lib.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, ctypes.byref(b), 2048, 64, 128)
    assert need >= 2 * 256 * 4 + 2 * 2048 * 4
    q = lib.dsa_quantize_index_keys
    assert q(None, 10, 128, 128, FAKE, FAKE, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert q(FAKE, 10, 128, 48, FAKE, FAKE, None) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert q(FAKE, 10, 100, 32, FAKE, FAKE, None) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert q(MIS, 10, 128, 128, FAKE, FAKE, None) == B.DSA_ERR_MISALIGNED
    assert q(FAKE, -1, 128, 128, FAKE, FAKE, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert q(FAKE, 0, 128, 128, FAKE, FAKE, None) == B.DSA_OK
    d = lib.dsa_dequantize_index_keys
    assert d(FAKE, FAKE, 10, 128, 96, FAKE, None) == B.DSA_ERR_UNSUPPORTED_SHAPE
    assert d(FAKE, FAKE, 0, 128, 128, FAKE, None) == B.DSA_OK


def test_workspace_sizes(lib):
    b = _batch(num_q=32, batch=32, max_seq_len=8192)
    # the indexer needs room only for MXFP8 queries widened to bf16 (T x H_I x d_I x 2 bytes)
    qb = 32 * 64 * 128 * 2
    assert lib.dsa_workspace_size(B.DSA_OP_INDEXER_SCORES, ctypes.byref(b), 2048, 64, 128) == qb
    assert lib.dsa_workspace_size(B.DSA_OP_TOPK, ctypes.byref(b), 2048, 64, 128) == 0
    fused = lib.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, ctypes.byref(b), 2048, 64, 128)
    mla = lib.dsa_workspace_size(B.DSA_OP_SPARSE_MLA, ctypes.byref(b), 2048, 64, 128)
    assert fused == 32 * 8192 * 4 + 32 * 2048 * 4 + mla + qb
    assert lib.dsa_workspace_size(B.DSA_OP_FUSED_DECODE, None, 2048, 64, 128) == 0


def test_attention_workspace_layout(lib):
    """The 128-head attention's workspace: four P slots (128 x 64 bf16 image +
    128 fp32 factors = 16896 B) and 128 (max, sum) pairs for each of 256 SM
    records, then, with S > 1 key splits, S x T x 128 partial rows of 512 fp32
    plus their (max, sum). The split count comes from the device's resident
    cluster count (or the SM count without a device): 1 to 4."""
    b = _batch(num_q=32, batch=32, max_seq_len=8192)
    mla = lib.dsa_workspace_size(B.DSA_OP_SPARSE_MLA, ctypes.byref(b), 2048, 64, 128)
    ring_fin = 256 * 4 * 16896 + 256 * 128 * 8
    per_split = 32 * 128 * (512 * 4 + 8)
    assert mla - ring_fin in (0, 2 * per_split, 3 * per_split, 4 * per_split)
    # one query: every split count up to 4 fits in one wave; 32 key tiles -> 4 splits
    b1 = _batch(num_q=1, batch=1, max_seq_len=8192)
    one = lib.dsa_workspace_size(B.DSA_OP_SPARSE_MLA, ctypes.byref(b1), 2048, 64, 128)
    assert one == ring_fin + 4 * 128 * (512 * 4 + 8)


def _header_shapes():
    """The supported-shape block of include/dsa.h, parsed."""
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    pairs = lambda line: {tuple(int(v) for v in m) for m in re.findall(r"\((\d+),\s*(\d+)\)", line)}
    idx_line = re.search(r"indexer \(H_I, d_I\):(.*)", text).group(1)
    mla_line = re.search(r"MLA \(d_latent, d_rope\):(.*)", text).group(1)
    heads_line = re.search(r"MLA heads H:(.*)", text).group(1)
    k_line = re.search(r"top-K k:(.*)", text).group(1)
    heads = set()
    for lo, hi in re.findall(r"(\d+)\.\.(\d+)", heads_line):
        heads |= set(range(int(lo), int(hi) + 1))
    heads |= {int(v) for v in re.findall(r"or (\d+)", heads_line)}
    k_lo, k_hi = (int(v) for v in re.search(r"(\d+)\.\.(\d+)", k_line).groups())
    return pairs(idx_line), pairs(mla_line), heads, (k_lo, k_hi)


def test_header_supported_shapes_match_validation(lib):
    """Every shape the header lists passes validation (an empty batch then
    returns DSA_OK with nothing enqueued) and every shape it does not list is
    rejected with DSA_ERR_UNSUPPORTED_SHAPE."""
    idx_pairs, mla_pairs, heads, (k_lo, k_hi) = _header_shapes()
    assert idx_pairs == {(4, 32), (4, 128), (64, 32), (64, 128)}
    empty = _batch(num_q=0)
    for hi in (1, 2, 4, 8, 16, 32, 48, 64, 96, 128):
        for di in (16, 32, 64, 96, 128, 256):
            want = B.DSA_OK if (hi, di) in idx_pairs else B.DSA_ERR_UNSUPPORTED_SHAPE
            assert _scores(lib, empty, _idx_in(n_heads=hi, head_dim=di, scale_group=di)) == want, (hi, di)
    for dl, dr in [(512, 64), (64, 16), (512, 0), (256, 64), (64, 64), (128, 16), (576, 0)]:
        for h in (1, 4, 32, 63, 64, 65, 96, 127, 128, 129, 192, 256):
            want = B.DSA_OK if ((dl, dr) in mla_pairs and h in heads) else B.DSA_ERR_UNSUPPORTED_SHAPE
            got = lib.dsa_sparse_mla_attn(ctypes.byref(empty), ctypes.byref(_mla_in(n_heads=h, d_latent=dl, d_rope=dr)),
                                          FAKE, 64, FAKE, None, None, 0, None)
            assert got == want, (dl, dr, h)
    for k in (k_lo - 1, k_lo, 2, 1024, k_hi, k_hi + 1):
        want = B.DSA_OK if k_lo <= k <= k_hi else B.DSA_ERR_UNSUPPORTED_SHAPE
        assert lib.dsa_topk(ctypes.byref(empty), FAKE, 256, k, FAKE, None, 0, None) == want, k
        got = lib.dsa_sparse_mla_attn(ctypes.byref(empty), ctypes.byref(_mla_in()), FAKE, k, FAKE, None, None, 0, None)
        assert got == want, k


def test_header_page_size_rule_matches_validation(lib):
    """The header's paged-cache line (a positive multiple of N) against validation."""
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    mult = int(re.search(r"paged caches: page_size a positive multiple of (\d+)", text).group(1))
    assert mult == 64
    for ps in (32, 64, 96, 128, 192, 256, 1000, 1024):
        want = B.DSA_OK if ps % mult == 0 else B.DSA_ERR_UNSUPPORTED_SHAPE
        b = _batch(num_q=0, block_table=FAKE, page_size=ps, num_pages=4)
        assert _scores(lib, b, _idx_in()) == want, ps


def test_delayed_copy_hook_validation(lib):
    """The ordering test hook rejects what it cannot copy before it launches
    anything: NULL pointers, addresses or sizes that are not multiples of 16
    bytes, and delays above one second."""
    h = lib.dsa_debug_delayed_copy
    assert h(None, FAKE, 64, 0, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert h(FAKE, None, 64, 0, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert h(MIS, FAKE, 64, 0, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert h(FAKE, FAKE, 60, 0, None) == B.DSA_ERR_INVALID_ARGUMENT
    assert h(FAKE, FAKE, 64, 1_000_000_001, None) == B.DSA_ERR_INVALID_ARGUMENT
