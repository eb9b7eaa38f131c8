"""Seeded synthetic inputs for the indexed sparse attention (DSA) hot path.

This module only draws numbers: it holds none of the method's arithmetic. Both
the CUDA path (through the bindings) and the CPU oracle consume the arrays it
returns, so the two sides always see bit-identical inputs.

Every floating-point tensor is drawn in fp32 and rounded to bfloat16 (round to
nearest even) before either side sees it; arrays are returned as fp32 holding
bf16-exact values, plus a uint16 view of the bf16 bits for the device copy.

Random streams are counter based (numpy Philox keyed by (seed, tensor tag),
counter = block number), so any block of rows can be regenerated on its own;
that is what lets a test regenerate only the rows it samples from a large
cache.

Workloads (shapes, seeds and value laws) follow the five configurations the
DSA hot path is measured on:

* ``c1``  tiny decode, 1 sequence, L=256, 4 queries at 252..255, integer values
  in [-3, 3] everywhere; H_I=4, d_I=32, K=32, 4 MLA heads, d_c=64, d_rope=16.
* ``c2``  decode, batch 32, L=8192, one query each; H_I=64, d_I=128, K=2048;
  128 MLA heads, d_c=512, d_rope=64; N(0,1) except w ~ N(0, 1/64).
* ``c3``  ragged decode, batch 64, lengths U[1024, 65536]; FP8 index keys.
* ``c4``  causal prefill, one 32768-token sequence.
* ``c5``  chunked prefill, 4 x (131072 prefix + 8192 chunk), FP8 index keys;
  ``c5i`` is its integer-valued variant (values in [-2, 2]).
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Workload", "bf16_round", "bf16_bits", "make", "CONFIGS", "scaled",
]

# Seeds: one per configuration (the configuration number; 51 for the integer
# variant of the chunked prefill).
_SEEDS = {"c1": 1, "c2": 2, "c3": 3, "c4": 4, "c5": 5, "c5i": 51}

# Rows per generation block (a block is one Philox stream).
_BLOCK_ROWS = 4096


def bf16_round(x: np.ndarray, inplace: bool = False) -> np.ndarray:
    """Round finite fp32 values to the nearest bfloat16 (ties to even); returns fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if not inplace:
        x = x.copy()
    u = x.view(np.uint32)
    r = u >> 16
    r &= 1
    r += 0x7FFF
    u += r                      # no overflow: finite values are below 0xFF800000
    u &= np.uint32(0xFFFF0000)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of fp32 values that are bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _key(seed: int, tag: str):
    return [seed & 0xFFFFFFFFFFFFFFFF, zlib.crc32(tag.encode()) & 0xFFFFFFFF]


def _stream(seed: int, tag: str, block: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=_key(seed, tag), counter=[block, 0, 0, 0]))


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        import concurrent.futures
        import os
        _POOL = concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1))
    return _POOL


def _draw_rows(seed: int, tag: str, n_rows: int, row_elems: int, law, row_blocks=None,
               round_bf16: bool = False) -> np.ndarray:
    """Draw an [n_rows, row_elems] fp32 array block by block (threads over blocks).

    ``law(gen, shape)`` draws one block. ``row_blocks`` optionally restricts the
    draw to the listed blocks (the others are left zero). ``round_bf16`` rounds
    each block to bfloat16 in place."""
    out = np.zeros((n_rows, row_elems), dtype=np.float32)
    n_blocks = (n_rows + _BLOCK_ROWS - 1) // _BLOCK_ROWS
    blocks = range(n_blocks) if row_blocks is None else sorted(set(row_blocks))

    def one(blk):
        r0 = blk * _BLOCK_ROWS
        r1 = min(n_rows, r0 + _BLOCK_ROWS)
        out[r0:r1] = law(_stream(seed, tag, blk), (r1 - r0, row_elems))
        if round_bf16:
            bf16_round(out[r0:r1], inplace=True)

    blocks = list(blocks)
    if len(blocks) > 1:
        list(_pool().map(one, blocks))
    else:
        for blk in blocks:
            one(blk)
    return out


def _normal(std: float):
    def law(g, shape):
        return g.standard_normal(shape, dtype=np.float32) * np.float32(std)
    return law


def _ints(lo: int, hi: int):
    def law(g, shape):
        return g.integers(lo, hi + 1, size=shape).astype(np.float32)
    return law


@dataclasses.dataclass
class Workload:
    """One synthetic instance of the DSA hot path.

    Layouts (row-major):
      cu_q [B+1] int32     query-token offsets per sequence
      q_pos [T] int32      position of each query token inside its sequence
      seq_lens [B] int32   valid cache rows per sequence
      q_idx [T,HI,dI]      indexer queries (bf16-exact fp32)
      w [T,HI]             head weights (fp32)
      k_idx [B,Lmax,dI]    index keys (bf16-exact fp32); quantised to FP8 by the
                           cache-write step when key_dtype == "fp8"
      q [T,H,D]            MLA queries, D = d_c + d_rope (bf16-exact fp32)
      kv [B,Lmax,D]        latent KV cache rows (bf16-exact fp32)
    """
    name: str
    B: int
    T: int
    Lmax: int
    cu_q: np.ndarray
    q_pos: np.ndarray
    seq_lens: np.ndarray
    HI: int
    dI: int
    H: int
    dc: int
    dr: int
    K: int
    key_dtype: str          # "bf16" | "fp8"
    scale_group: int        # FP8 scale group (elements per scale)
    softmax_scale: float
    q_idx: np.ndarray
    w: np.ndarray
    k_idx: Optional[np.ndarray]
    q: np.ndarray
    kv: Optional[np.ndarray]
    seed: int
    integer_valued: bool
    laws: dict = dataclasses.field(default_factory=dict, repr=False)  # cache tag -> value law
    seq_ids: Optional[np.ndarray] = None  # sequences of a parent workload these are (select_sequences)

    @property
    def D(self) -> int:
        return self.dc + self.dr

    def seq_of_token(self) -> np.ndarray:
        """Sequence id of every query token (from cu_q)."""
        return (np.searchsorted(self.cu_q, np.arange(self.T), side="right") - 1).astype(np.int32)

    def n_valid(self) -> np.ndarray:
        """Causal candidate count per query: min(pos + 1, len of its sequence)."""
        b = self.seq_of_token()
        return np.minimum(self.q_pos + 1, self.seq_lens[b]).astype(np.int32)

    def seq_rows(self, tag: str, b: int) -> np.ndarray:
        """Cache rows [seq_len_b, dim] of sequence b (tag 'k_idx' or 'kv'), regenerated
        from the same counter-based streams the full cache is drawn from."""
        dim = self.dI if tag == "k_idx" else self.D
        src = b if self.seq_ids is None else int(self.seq_ids[b])
        return _draw_rows(self.seed, f"{tag}/{src}", int(self.seq_lens[b]), dim, self.laws[tag], round_bf16=True)


def _cache(seed, tag, B, Lmax, lens, dim, law, rows_needed=None):
    """A [B, Lmax, dim] cache; rows at or beyond a sequence's length are zero.

    ``rows_needed`` (dict b -> iterable of rows) restricts generation to the
    blocks holding those rows (for sampled checks on very large caches)."""
    out = np.zeros((B, Lmax, dim), dtype=np.float32)
    for b in range(B):
        n = int(lens[b])
        blocks = None
        if rows_needed is not None:
            rows = rows_needed.get(b, ())
            blocks = {int(r) // _BLOCK_ROWS for r in rows}
            if not blocks:
                continue
        out[b, :n] = _draw_rows(seed, f"{tag}/{b}", n, dim, law, blocks, round_bf16=True)
    return out


def make(name: str, *, with_caches: bool = True, rows_needed: Optional[Dict[int, list]] = None,
         tokens: Optional[slice] = None, queries: bool = True) -> Workload:
    """Build the synthetic workload ``name`` (see the module docstring).

    ``with_caches=False`` skips drawing the two caches (k_idx, kv).
    ``rows_needed`` limits cache generation to the blocks holding those rows.
    ``queries=False`` skips drawing the query tensors too (shapes and laws
    only: q_idx, w and q are left empty).
    """
    seed = _SEEDS[name]
    if name == "c1":
        B, Lmax, HI, dI, H, dc, dr, K = 1, 256, 4, 32, 4, 64, 16, 32
        lens = np.array([256], np.int32)
        cu_q = np.array([0, 4], np.int32)
        q_pos = np.array([252, 253, 254, 255], np.int32)
        law_q = law_k = law_w = law_mla = _ints(-3, 3)
        key_dtype, integer = "bf16", True
    elif name == "c2":
        B, Lmax, HI, dI, H, dc, dr, K = 32, 8192, 64, 128, 128, 512, 64, 2048
        lens = np.full(B, 8192, np.int32)
        cu_q = np.arange(B + 1, dtype=np.int32)
        q_pos = lens - 1
        law_q = law_k = law_mla = _normal(1.0)
        law_w = _normal(1.0 / 8.0)
        key_dtype, integer = "bf16", False
    elif name == "c3":
        B, Lmax, HI, dI, H, dc, dr, K = 64, 65536, 64, 128, 128, 512, 64, 2048
        g = _stream(seed, "seq_lens", 0)
        lens = g.integers(1024, 65536 + 1, size=B).astype(np.int32)
        cu_q = np.arange(B + 1, dtype=np.int32)
        q_pos = lens - 1
        law_q = law_k = law_mla = _normal(1.0)
        law_w = _normal(1.0 / 8.0)
        key_dtype, integer = "fp8", False
    elif name == "c4":
        B, Lmax, HI, dI, H, dc, dr, K = 1, 32768, 64, 128, 128, 512, 64, 2048
        lens = np.array([32768], np.int32)
        cu_q = np.array([0, 32768], np.int32)
        q_pos = np.arange(32768, dtype=np.int32)
        law_q = law_k = law_mla = _normal(1.0)
        law_w = _normal(1.0 / 8.0)
        key_dtype, integer = "bf16", False
    elif name in ("c5", "c5i"):
        B, HI, dI, H, dc, dr, K = 4, 64, 128, 128, 512, 64, 2048
        prefix, chunk = 131072, 8192
        Lmax = prefix + chunk
        lens = np.full(B, Lmax, np.int32)
        cu_q = (np.arange(B + 1) * chunk).astype(np.int32)
        q_pos = np.tile(np.arange(prefix, prefix + chunk, dtype=np.int32), B)
        if name == "c5":
            law_q = law_k = law_mla = _normal(1.0)
            law_w = _normal(1.0 / 8.0)
            integer = False
        else:
            law_q = law_k = law_w = law_mla = _ints(-2, 2)
            integer = True
        key_dtype = "fp8"
    else:
        raise KeyError(name)

    T = int(cu_q[-1])
    D = dc + dr
    if queries:
        q_idx = bf16_round(_draw_rows(seed, "q_idx", T, HI * dI, law_q)).reshape(T, HI, dI)
        w = _draw_rows(seed, "w", T, HI, law_w).astype(np.float32)
        q = bf16_round(_draw_rows(seed, "q", T, H * D, law_mla)).reshape(T, H, D)
    else:
        q_idx = np.zeros((0, HI, dI), np.float32)
        w = np.zeros((0, HI), np.float32)
        q = np.zeros((0, H, D), np.float32)
    k_idx = kv = None
    if with_caches:
        k_idx = _cache(seed, "k_idx", B, Lmax, lens, dI, law_k, rows_needed)
        kv = _cache(seed, "kv", B, Lmax, lens, D, law_mla, rows_needed)
    wl = Workload(name=name, B=B, T=T, Lmax=Lmax, cu_q=cu_q, q_pos=q_pos.astype(np.int32),
                  seq_lens=lens.astype(np.int32), HI=HI, dI=dI, H=H, dc=dc, dr=dr, K=K,
                  key_dtype=key_dtype, scale_group=128 if dI >= 128 else dI,
                  softmax_scale=float(1.0 / np.sqrt(D)), q_idx=q_idx, w=w, k_idx=k_idx, q=q, kv=kv,
                  seed=seed, integer_valued=integer, laws={"k_idx": law_k, "kv": law_mla})
    if tokens is not None:
        wl = _select_tokens(wl, tokens)
    return wl


def _select_tokens(wl: Workload, tokens: slice) -> Workload:
    """Keep a contiguous range of query tokens (all within their sequences)."""
    idx = np.arange(wl.T)[tokens]
    b = wl.seq_of_token()[idx]
    counts = np.bincount(b, minlength=wl.B)
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return dataclasses.replace(wl, T=len(idx), cu_q=cu, q_pos=wl.q_pos[idx].copy(),
                               q_idx=wl.q_idx[idx].copy(), w=wl.w[idx].copy(), q=wl.q[idx].copy())


def scaled(name: str, *, B: int, Lmax: int, T_per_seq: int = 1, lens=None, K: Optional[int] = None,
           HI=None, dI=None, H=None, dc=None, dr=None, key_dtype=None, integer=None, seed=None) -> Workload:
    """A smaller instance with the value laws and head shapes of ``name``.

    Used by the parity tests: sizes the oracle finishes in seconds that still
    span several tiles and a ragged tail. Queries are the last ``T_per_seq``
    positions of every sequence."""
    base = make(name, with_caches=False, queries=False)
    HI = base.HI if HI is None else HI
    dI = base.dI if dI is None else dI
    H = base.H if H is None else H
    dc = base.dc if dc is None else dc
    dr = base.dr if dr is None else dr
    K = base.K if K is None else K
    key_dtype = base.key_dtype if key_dtype is None else key_dtype
    integer = base.integer_valued if integer is None else integer
    seed = (base.seed * 1000 + 7) if seed is None else seed
    if lens is None:
        lens = np.full(B, Lmax, np.int32)
    lens = np.asarray(lens, np.int32)
    tps = np.minimum(T_per_seq, lens)
    cu_q = np.concatenate([[0], np.cumsum(tps)]).astype(np.int32)
    q_pos = np.concatenate([np.arange(int(n) - int(k), int(n)) for n, k in zip(lens, tps)]).astype(np.int32)
    T = int(cu_q[-1])
    D = dc + dr
    if integer:
        lim = 3 if name == "c1" else 2
        law_q = law_k = law_w = law_mla = _ints(-lim, lim)
    else:
        law_q = law_k = law_mla = _normal(1.0)
        law_w = _normal(1.0 / 8.0)
    q_idx = bf16_round(_draw_rows(seed, "q_idx", T, HI * dI, law_q)).reshape(T, HI, dI)
    w = _draw_rows(seed, "w", T, HI, law_w).astype(np.float32)
    q = bf16_round(_draw_rows(seed, "q", T, H * D, law_mla)).reshape(T, H, D)
    k_idx = _cache(seed, "k_idx", B, Lmax, lens, dI, law_k)
    kv = _cache(seed, "kv", B, Lmax, lens, D, law_mla)
    return Workload(name=f"{name}-scaled", B=B, T=T, Lmax=Lmax, cu_q=cu_q, q_pos=q_pos, seq_lens=lens,
                    HI=HI, dI=dI, H=H, dc=dc, dr=dr, K=K, key_dtype=key_dtype,
                    scale_group=128 if dI >= 128 else dI, softmax_scale=float(1.0 / np.sqrt(D)),
                    q_idx=q_idx, w=w, k_idx=k_idx, q=q, kv=kv, seed=seed, integer_valued=integer,
                    laws={"k_idx": law_k, "kv": law_mla})


def restrict(wl: Workload, rows) -> Workload:
    """The workload seen by the query tokens ``rows`` only: their sequences
    (renumbered, in order), caches regenerated for those sequences alone, and
    Lmax cut to the longest of them. Values are identical to the full
    workload's: used to run the oracle on sampled rows of very large caches."""
    rows = np.asarray(rows, np.int64)
    seqs = np.unique(wl.seq_of_token()[rows])
    remap = {int(b): i for i, b in enumerate(seqs)}
    lens = wl.seq_lens[seqs].astype(np.int32)
    Lmax = int(lens.max())
    bt = np.array([remap[int(b)] for b in wl.seq_of_token()[rows]], np.int32)
    order = np.argsort(bt, kind="stable")
    rows, bt = rows[order], bt[order]
    counts = np.bincount(bt, minlength=len(seqs))
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    k_idx = np.zeros((len(seqs), Lmax, wl.dI), np.float32)
    kv = np.zeros((len(seqs), Lmax, wl.D), np.float32)
    for i, b in enumerate(seqs):
        n = int(wl.seq_lens[b])
        k_idx[i, :n] = wl.seq_rows("k_idx", int(b))
        kv[i, :n] = wl.seq_rows("kv", int(b))
    return dataclasses.replace(wl, B=len(seqs), T=len(rows), Lmax=Lmax, cu_q=cu, q_pos=wl.q_pos[rows].copy(),
                               seq_lens=lens, q_idx=wl.q_idx[rows].copy(), w=wl.w[rows].copy(),
                               q=wl.q[rows].copy(), k_idx=k_idx, kv=kv), rows


def select_sequences(wl: Workload, seqs) -> Workload:
    """The sequences ``seqs`` (ascending) of a workload made without host caches,
    with all their query tokens: the share of one rank when a batch of
    independent sequences is split across GPUs. Cache rows are regenerated
    from the parent's streams (seq_ids), so values are identical."""
    seqs = np.asarray(sorted(int(b) for b in seqs), np.int64)
    assert wl.k_idx is None and wl.kv is None, "select_sequences works on workloads made without host caches"
    b_of = wl.seq_of_token()
    rows = np.nonzero(np.isin(b_of, seqs))[0]
    counts = np.array([int(wl.cu_q[b + 1] - wl.cu_q[b]) for b in seqs], np.int64)
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    parent = wl.seq_ids if wl.seq_ids is not None else np.arange(wl.B)
    return dataclasses.replace(wl, B=len(seqs), T=len(rows), cu_q=cu, q_pos=wl.q_pos[rows].copy(),
                               seq_lens=wl.seq_lens[seqs].astype(np.int32), q_idx=wl.q_idx[rows].copy(),
                               w=wl.w[rows].copy(), q=wl.q[rows].copy(), seq_ids=parent[seqs].copy())


CONFIGS = tuple(_SEEDS)


def page_layout(seq_lens, Lmax: int, page_size: int, seed: int, spare_pages: int = 3):
    """A seeded random placement of every sequence's cache pages in one pool.

    Sequence b needs ceil(seq_lens[b] / page_size) pages; they get distinct
    pool pages drawn in random order from a pool with ``spare_pages`` pages
    nobody uses. Returns (block_table [B, ceil(Lmax / page_size)] int32, with
    -1 in every entry a sequence does not need, num_pages).
    """
    lens = np.asarray(seq_lens, np.int64)
    max_pages = (Lmax + page_size - 1) // page_size
    need = (lens + page_size - 1) // page_size
    num_pages = int(need.sum()) + spare_pages
    order = np.random.Generator(np.random.Philox(key=_key(seed, "pages"))).permutation(num_pages)
    table = np.full((len(lens), max_pages), -1, np.int32)
    pos = 0
    for b, n in enumerate(need):
        table[b, :n] = order[pos:pos + n]
        pos += int(n)
    return table, num_pages
