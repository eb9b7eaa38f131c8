"""fp64 CPU oracle for the indexed sparse attention (DSA) hot path.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package. The product path (the CUDA
library and its Python binding) never imports, loads or calls it, and the two
share no code: the only common module is the seeded input generator, which
holds none of the method's arithmetic.

The arithmetic lives in ``dsa_oracle.c`` (plain C, fp64, OpenMP over rows);
this module builds it with gcc on first use and wraps it with numpy.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.oracle_e4m3_decode.restype = ctypes.c_double
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_encode_satfinite.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode_satfinite.argtypes = [ctypes.c_float]
            lib.oracle_quantize_keys.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _u8p, _f32p]
            lib.oracle_dequantize_keys.argtypes = [_u8p, _f32p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _f32p]
            lib.oracle_indexer_scores.argtypes = [
                ctypes.c_int32, ctypes.c_int32, _i32p, _i32p, _i32p, ctypes.c_int32, ctypes.c_int32,
                _f32p, _f32p, ctypes.c_int32, _f32p, _u8p, _f32p, ctypes.c_int32,
                ctypes.c_int32, _i32p, _f64p, ctypes.c_int64]
            lib.oracle_topk.argtypes = [ctypes.c_int32, _f64p, ctypes.c_int64, _i32p, ctypes.c_int32, _i32p]
            lib.oracle_sparse_mla.argtypes = [
                ctypes.c_int32, ctypes.c_int32, _i32p, _i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                ctypes.c_double, _f32p, _f64p, ctypes.c_int32, _i32p, _i32p, ctypes.c_int32, _f64p, _f64p]
            lib.oracle_num_threads.restype = ctypes.c_int32
            lib.oracle_set_num_threads.argtypes = [ctypes.c_int32]
            _lib = lib
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def e4m3_decode(codes) -> np.ndarray:
    """Decode E4M3 codes (uint8 array) to fp64 per the OCP FP8 definition."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_decode(int(v)) for v in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    """Round fp32 values to E4M3 codes (nearest-even, saturating to +-448)."""
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.oracle_e4m3_encode_satfinite(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def quantize_keys(k: np.ndarray, group: int):
    """Per-group FP8 cache write of keys [..., dim] -> (codes uint8, scales fp32)."""
    k = _c(k, np.float32)
    dim = k.shape[-1]
    n = k.size // dim
    codes = np.empty(k.shape, np.uint8)
    scales = np.empty(k.shape[:-1] + (dim // group,), np.float32)
    _load().oracle_quantize_keys(_p(k, _f32p), n, dim, group, _p(codes, _u8p), _p(scales, _f32p))
    return codes, scales


def dequantize_keys(codes: np.ndarray, scales: np.ndarray, group: int) -> np.ndarray:
    """fl32(decode(code) * scale) per element."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    dim = codes.shape[-1]
    n = codes.size // dim
    out = np.empty(codes.shape, np.float32)
    _load().oracle_dequantize_keys(_p(codes, _u8p), _p(scales, _f32p), n, dim, group, _p(out, _f32p))
    return out


def indexer_scores(wl, rows=None, *, k_codes=None, k_scales=None) -> np.ndarray:
    """Oracle scores [len(rows), Lmax] (fp64; -inf where masked) for workload ``wl``.

    FP8 keys are used when ``k_codes``/``k_scales`` are given (dequantised in
    fp64 inside the oracle); otherwise the bf16 keys ``wl.k_idx``."""
    lib = _load()
    rows = np.arange(wl.T, dtype=np.int32) if rows is None else _c(rows, np.int32)
    out = np.empty((len(rows), wl.Lmax), np.float64)
    cu_q, q_pos, lens = _c(wl.cu_q, np.int32), _c(wl.q_pos, np.int32), _c(wl.seq_lens, np.int32)
    q_idx, w = _c(wl.q_idx, np.float32), _c(wl.w, np.float32)
    if k_codes is not None:
        k8, ks = _c(k_codes, np.uint8), _c(k_scales, np.float32)
        kf = np.zeros(1, np.float32)
        is8 = 1
        group = wl.dI // ks.shape[-1]
    else:
        kf = _c(wl.k_idx, np.float32)
        k8, ks = np.zeros(1, np.uint8), np.zeros(1, np.float32)
        is8 = 0
        group = wl.dI
    lib.oracle_indexer_scores(wl.B, wl.Lmax, _p(cu_q, _i32p), _p(q_pos, _i32p), _p(lens, _i32p),
                              wl.HI, wl.dI, _p(q_idx, _f32p), _p(w, _f32p), is8, _p(kf, _f32p),
                              _p(k8, _u8p), _p(ks, _f32p), group, len(rows), _p(rows, _i32p),
                              _p(out, _f64p), wl.Lmax)
    return out


def topk(scores: np.ndarray, n_valid, K: int) -> np.ndarray:
    """Top-K positions per row (ties: higher score, then lower position);
    ascending by position, padded with -1."""
    s = _c(scores, np.float64)
    nv = _c(n_valid, np.int32)
    out = np.empty((s.shape[0], K), np.int32)
    _load().oracle_topk(s.shape[0], _p(s, _f64p), s.shape[1], _p(nv, _i32p), K, _p(out, _i32p))
    return out


def sparse_mla(wl, idx: np.ndarray, rows=None, kv=None):
    """Attention over the selected rows: returns (out [n,H,dc] fp64, lse [n,H] fp64).

    ``kv`` replaces the workload's bf16 latent rows (e.g. the FP8 cache's
    rows dequantised in fp64 by :func:`dequantize_kv`)."""
    lib = _load()
    rows = np.arange(wl.T, dtype=np.int32) if rows is None else _c(rows, np.int32)
    idx = _c(idx, np.int32)
    K = idx.shape[1]
    out = np.empty((len(rows), wl.H, wl.dc), np.float64)
    lse = np.empty((len(rows), wl.H), np.float64)
    cu_q, lens = _c(wl.cu_q, np.int32), _c(wl.seq_lens, np.int32)
    q = _c(wl.q, np.float32)
    kv = _c(wl.kv if kv is None else kv, np.float64)
    lib.oracle_sparse_mla(wl.B, wl.Lmax, _p(cu_q, _i32p), _p(lens, _i32p), wl.H, wl.D, wl.dc,
                          float(wl.softmax_scale), _p(q, _f32p), _p(kv, _f64p), len(rows),
                          _p(rows, _i32p), _p(idx, _i32p), K, _p(out, _f64p), _p(lse, _f64p))
    return out, lse


def dsa(wl, rows=None, *, k_codes=None, k_scales=None, rank_in_fp32: bool = False):
    """The whole hot path for the rows ``rows``: (scores, idx, out, lse).

    ``rank_in_fp32`` ranks the fp64 scores after one rounding to fp32, the
    precision in which the kernel takes the Top-K decision (used where the
    scores are exact integers times one fp32 scale)."""
    rows = np.arange(wl.T, dtype=np.int32) if rows is None else np.asarray(rows, np.int32)
    sc = indexer_scores(wl, rows, k_codes=k_codes, k_scales=k_scales)
    rank = sc.astype(np.float32).astype(np.float64) if rank_in_fp32 else sc
    nv = wl.n_valid()[rows]
    idx = topk(rank, nv, wl.K)
    out, lse = sparse_mla(wl, idx, rows)
    return sc, idx, out, lse


def unpage(pool: np.ndarray, block_table: np.ndarray, page_size: int, Lmax: int) -> np.ndarray:
    """The logical cache [B, Lmax, ...] of a page pool [num_pages * page_size, ...].

    Paged caches (the fused indexer reads the paged key cache directly:
    section 3 of "Optimizing Inference for New Model Architectures ..."):
    row s of sequence b is pool row
        block_table[b, s // page_size] * page_size + s % page_size.
    Rows of a page whose table entry is -1 are zero. Plain loops over rows
    (small cases only)."""
    pool = np.asarray(pool)
    table = np.asarray(block_table)
    out = np.zeros((table.shape[0], Lmax) + pool.shape[1:], pool.dtype)
    for b in range(table.shape[0]):
        for s in range(Lmax):
            pg = int(table[b, s // page_size])
            if pg >= 0:
                out[b, s] = pool[pg * page_size + s % page_size]
    return out


def quantize_kv(kv: np.ndarray, dc: int, tile: int = 128):
    """FP8 cache write of latent KV rows [..., dc + d_rope] (Block-Wise
    Quantization for Key-Value Cache: "Optimizing Inference for New Model
    Architectures ...", section 4; Tiered Quantization table of "Day-0
    Inference Adaptation ..."): the dc latent dims in tiles of ``tile``
    elements (one tile when dc < tile), each with scale = absmax / 448 and
    codes e4m3(round to nearest even, saturating)(x / scale) -- the same
    per-group dynamic quantisation as the index keys; the rope dims stay bf16.
    Returns (codes [..., dc] uint8, scales [..., dc / g] fp32, rope [..., d_rope] fp32)."""
    kv = _c(kv, np.float32)
    g = min(tile, dc)
    codes, scales = quantize_keys(np.ascontiguousarray(kv[..., :dc]), g)
    return codes, scales, np.ascontiguousarray(kv[..., dc:])


def dequantize_kv(codes: np.ndarray, scales: np.ndarray, rope: np.ndarray) -> np.ndarray:
    """fp64 latent rows of an FP8 KV cache: decode(code) * tile scale (exact in
    fp64: a code carries 4 significant bits, a scale 24), then the rope dims."""
    g = codes.shape[-1] // scales.shape[-1]
    lat = e4m3_decode(codes) * np.repeat(np.asarray(scales, np.float64), g, axis=-1)
    return np.concatenate([lat, np.asarray(rope, np.float64)], axis=-1)


def mx_quantize(x: np.ndarray, group: int = 32):
    """MXFP8 per-group dynamic quantisation of index queries / keys [..., dim]
    (Index Q/K Uses MXFP8, section 4.2 of "Inference Adaptation and
    Performance Optimization for New Large Language Model Architectures";
    every 32 elements share one scale factor).

    Reading: the group's scale is the per-group pseudocode's absmax / 448
    rounded up to a power of two 2^e -- the E8M0 shared scale of the MX
    format, chosen so that no element saturates: e is the least integer
    with 448 * 2^e >= absmax (an exact comparison), kept in [-127, 127];
    absmax = 0 gives e = -127 and codes 0. Each element's code is the E4M3
    cast (nearest even, saturating) of x / 2^e, which is exact before the
    cast. Returns (codes uint8 [..., dim], scale bytes uint8 [..., dim / group]
    holding e + 127)."""
    x = np.asarray(x, np.float32)
    dim = x.shape[-1]
    g = x.reshape(-1, dim // group, group).astype(np.float64)
    amax = np.abs(g).max(axis=-1)
    e = np.full(amax.shape, -127, np.int64)
    nz = amax > 0
    e[nz] = np.floor(np.log2(amax[nz] / 448.0)).astype(np.int64) - 1
    for _ in range(4):  # settle on the least e with 448 * 2^e >= absmax (exact in fp64)
        up = nz & (448.0 * np.ldexp(1.0, e) < amax)
        e[up] += 1
    down = nz & (448.0 * np.ldexp(1.0, e - 1) >= amax)
    assert not down.any()
    e = np.clip(e, -127, 127)
    scaled = (g * np.ldexp(1.0, -e)[..., None]).astype(np.float32)
    codes = e4m3_encode(scaled).reshape(x.shape)
    return codes, (e + 127).astype(np.uint8).reshape(x.shape[:-1] + (dim // group,))


def mx_dequantize(codes: np.ndarray, scale_bytes: np.ndarray) -> np.ndarray:
    """decode(code) * 2^(byte - 127), exact (fp64; also exact in fp32 and
    bf16 while the result stays inside their normal range)."""
    g = codes.shape[-1] // scale_bytes.shape[-1]
    e = np.repeat(np.asarray(scale_bytes, np.int64) - 127, g, axis=-1)
    return e4m3_decode(codes) * np.ldexp(1.0, e)
