"""Thin ctypes binding of libdsa.so (the C ABI in include/dsa.h).

Argument marshalling only: every step of the DSA hot path runs in the CUDA
kernels behind these calls. PyTorch supplies device memory and streams. The
library must be built (``python -m indexed_sparse_attention_relu_b200.build``);
there is no fallback of any kind: a missing library raises.

The functions carry the C names (dsa_indexer_scores, dsa_topk,
dsa_sparse_mla_attn, dsa_fused_decode, dsa_quantize_index_keys,
dsa_dequantize_index_keys, dsa_workspace_size, dsa_read_device_status) and
take the ctypes structs below plus torch tensors for the buffers.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_void_p

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARGUMENT = 1
DSA_ERR_UNSUPPORTED_SHAPE = 2
DSA_ERR_WORKSPACE_TOO_SMALL = 3
DSA_ERR_CUDA = 4
DSA_ERR_DEVICE_INDEX = 5
DSA_ERR_DEVICE_TIMEOUT = 6
DSA_ERR_MISALIGNED = 7
DSA_ERR_DEVICE_LAYOUT = 8

DSA_KEY_BF16 = 0
DSA_KEY_FP8_E4M3 = 1
DSA_KEY_MXFP8 = 2
DSA_KV_BF16 = 0
DSA_KV_FP8_E4M3 = 1

DSA_OP_INDEXER_SCORES = 0
DSA_OP_TOPK = 1
DSA_OP_SPARSE_MLA = 2
DSA_OP_FUSED_DECODE = 3

# Every symbol include/dsa.h declares.
EXPORTED = (
    "dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_fused_decode", "dsa_fused_decode_noalloc",
    "dsa_quantize_index_keys", "dsa_dequantize_index_keys", "dsa_quantize_kv", "dsa_kv_fp8_row_bytes",
    "dsa_quantize_mxfp8",
    "dsa_workspace_size",
    "dsa_read_device_status", "dsa_status_string", "dsa_last_error", "dsa_version",
    "dsa_debug_set_wait_limit", "dsa_debug_withhold_signal", "dsa_debug_delayed_copy",
)


class DsaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{status_string(status)} ({status}): {detail}")
        self.status = status


class dsa_batch(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("num_q", c_int32), ("max_seq_len", c_int32),
                ("cu_q", c_void_p), ("q_pos", c_void_p), ("seq_lens", c_void_p),
                ("block_table", c_void_p), ("page_size", c_int32), ("num_pages", c_int32)]


class dsa_indexer_in(ctypes.Structure):
    _fields_ = [("n_heads", c_int32), ("head_dim", c_int32), ("q", c_void_p), ("w", c_void_p),
                ("key_dtype", c_int32), ("k_cache", c_void_p), ("k_scale", c_void_p), ("scale_group", c_int32),
                ("q_scale_e8m0", c_void_p), ("k_scale_e8m0", c_void_p)]


class dsa_mla_in(ctypes.Structure):
    _fields_ = [("n_heads", c_int32), ("d_latent", c_int32), ("d_rope", c_int32), ("softmax_scale", c_float),
                ("q", c_void_p), ("kv", c_void_p), ("kv_dtype", c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m indexed_sparse_attention_relu_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P = c_void_p
        sig = {
            "dsa_indexer_scores": (c_int, [POINTER(dsa_batch), POINTER(dsa_indexer_in), P, c_int64, P, c_size_t, P]),
            "dsa_topk": (c_int, [POINTER(dsa_batch), P, c_int64, c_int32, P, P, c_size_t, P]),
            "dsa_sparse_mla_attn": (c_int, [POINTER(dsa_batch), POINTER(dsa_mla_in), P, c_int32, P, P, P, c_size_t, P]),
            "dsa_fused_decode": (c_int, [POINTER(dsa_batch), POINTER(dsa_indexer_in), POINTER(dsa_mla_in), c_int32,
                                         P, P, P, P, c_size_t, P, P]),
            "dsa_fused_decode_noalloc": (c_int, [POINTER(dsa_batch), POINTER(dsa_indexer_in), POINTER(dsa_mla_in),
                                                 c_int32, P, P, P, P]),
            "dsa_quantize_index_keys": (c_int, [P, c_int64, c_int32, c_int32, P, P, P]),
            "dsa_dequantize_index_keys": (c_int, [P, P, c_int64, c_int32, c_int32, P, P]),
            "dsa_quantize_kv": (c_int, [P, c_int64, c_int32, c_int32, P, P]),
            "dsa_quantize_mxfp8": (c_int, [P, c_int64, c_int32, P, P, P]),
            "dsa_kv_fp8_row_bytes": (c_size_t, [c_int32, c_int32]),
            "dsa_workspace_size": (c_size_t, [c_int, POINTER(dsa_batch), c_int32, c_int32, c_int32]),
            "dsa_read_device_status": (c_int, [P, POINTER(c_int32)]),
            "dsa_status_string": (c_char_p, [c_int]),
            "dsa_last_error": (c_char_p, []),
            "dsa_version": (c_char_p, []),
            "dsa_debug_set_wait_limit": (c_int, [ctypes.c_uint64]),
            "dsa_debug_withhold_signal": (c_int, [c_int32]),
            "dsa_debug_delayed_copy": (c_int, [P, P, c_size_t, ctypes.c_uint64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().dsa_status_string(status).decode()


def last_error() -> str:
    return load().dsa_last_error().decode()


def _check(status: int) -> None:
    if status != DSA_OK:
        raise DsaError(status, last_error())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ----------------------------------------------------------------------------- struct builders

class Batch:
    """Owns the int32 metadata tensors and exposes the dsa_batch struct.
    ``block_table`` ([B, ceil(max_seq_len / page_size)] int32), ``page_size``
    and ``num_pages`` describe paged caches; all None/0 for contiguous ones."""

    def __init__(self, cu_q: torch.Tensor, q_pos: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                 block_table: torch.Tensor | None = None, page_size: int = 0, num_pages: int = 0):
        self.cu_q, self.q_pos, self.seq_lens, self.block_table = cu_q, q_pos, seq_lens, block_table
        self.struct = dsa_batch(seq_lens.numel(), q_pos.numel(), int(max_seq_len), _ptr(cu_q), _ptr(q_pos),
                                _ptr(seq_lens), _ptr(block_table), int(page_size), int(num_pages))

    @property
    def ref(self):
        return ctypes.byref(self.struct)


def indexer_in(q: torch.Tensor, w: torch.Tensor, k_cache: torch.Tensor, k_scale: torch.Tensor | None = None,
               scale_group: int | None = None, q_mx: torch.Tensor | None = None,
               k_mx: torch.Tensor | None = None) -> dsa_indexer_in:
    """BF16 keys; FP8 keys (uint8 codes + fp32 ``k_scale``); or MXFP8 queries
    and keys (uint8 codes for both, E8M0 bytes ``q_mx`` / ``k_mx``)."""
    T, HI, DI = q.shape
    if q_mx is not None:
        return dsa_indexer_in(HI, DI, _ptr(q), _ptr(w), DSA_KEY_MXFP8, _ptr(k_cache), None, 32, _ptr(q_mx),
                              _ptr(k_mx))
    fp8 = k_cache.dtype in (torch.uint8, torch.float8_e4m3fn)
    return dsa_indexer_in(HI, DI, _ptr(q), _ptr(w), DSA_KEY_FP8_E4M3 if fp8 else DSA_KEY_BF16, _ptr(k_cache),
                          _ptr(k_scale), int(scale_group if scale_group is not None else DI), None, None)


def mla_in(q: torch.Tensor, kv: torch.Tensor, d_latent: int, softmax_scale: float) -> dsa_mla_in:
    """bf16 latent rows, or packed FP8 rows (a uint8 tensor written by
    dsa_quantize_kv)."""
    T, H, D = q.shape
    fp8 = kv.dtype == torch.uint8
    return dsa_mla_in(H, int(d_latent), int(D - d_latent), float(softmax_scale), _ptr(q), _ptr(kv),
                      DSA_KV_FP8_E4M3 if fp8 else DSA_KV_BF16)


# ----------------------------------------------------------------------------- C-ABI calls

def dsa_workspace_size(op: int, batch: Batch, k: int, h_i: int = 64, d_i: int = 128) -> int:
    return int(load().dsa_workspace_size(op, batch.ref, k, h_i, d_i))


def dsa_indexer_scores(batch: Batch, inp: dsa_indexer_in, scores: torch.Tensor, score_ld: int | None = None,
                       ws=None, ws_bytes: int = 0, stream=None) -> None:
    ld = scores.shape[-1] if score_ld is None else score_ld
    _check(load().dsa_indexer_scores(batch.ref, ctypes.byref(inp), _ptr(scores), ld, _ptr(ws), ws_bytes,
                                     _stream(stream)))


def dsa_topk(batch: Batch, scores: torch.Tensor, k: int, idx: torch.Tensor, score_ld: int | None = None,
             ws=None, ws_bytes: int = 0, stream=None) -> None:
    ld = scores.shape[-1] if score_ld is None else score_ld
    _check(load().dsa_topk(batch.ref, _ptr(scores), ld, k, _ptr(idx), _ptr(ws), ws_bytes, _stream(stream)))


def dsa_sparse_mla_attn(batch: Batch, inp: dsa_mla_in, idx: torch.Tensor, k: int, out: torch.Tensor,
                        lse: torch.Tensor | None = None, ws=None, ws_bytes: int | None = None, stream=None) -> None:
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(load().dsa_sparse_mla_attn(batch.ref, ctypes.byref(inp), _ptr(idx), k, _ptr(out), _ptr(lse), _ptr(ws),
                                      ws_bytes, _stream(stream)))


def dsa_fused_decode(batch: Batch, idx_inp: dsa_indexer_in, mla_inp: dsa_mla_in, k: int, out: torch.Tensor,
                     lse: torch.Tensor | None = None, idx_out: torch.Tensor | None = None, ws=None,
                     ws_bytes: int | None = None, stage_events=None, stream=None) -> None:
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    ev = None
    if stage_events is not None:
        for e in stage_events:
            if not e.cuda_event:          # torch creates the CUDA event on first record
                e.record(torch.cuda.current_stream() if stream is None else stream)
        arr = (c_void_p * 4)(*[e.cuda_event for e in stage_events])
        ev = ctypes.cast(arr, c_void_p)
    _check(load().dsa_fused_decode(batch.ref, ctypes.byref(idx_inp), ctypes.byref(mla_inp), k, _ptr(out), _ptr(lse),
                                   _ptr(idx_out), _ptr(ws), ws_bytes, ev, _stream(stream)))


def dsa_fused_decode_noalloc(batch: Batch, idx_inp: dsa_indexer_in, mla_inp: dsa_mla_in, k: int,
                             out: torch.Tensor, lse: torch.Tensor | None = None, idx_out: torch.Tensor | None = None,
                             stream=None) -> None:
    """The decode chain with the library's built-in scratch (no workspace)."""
    _check(load().dsa_fused_decode_noalloc(batch.ref, ctypes.byref(idx_inp), ctypes.byref(mla_inp), k, _ptr(out),
                                           _ptr(lse), _ptr(idx_out), _stream(stream)))


def dsa_quantize_index_keys(k_bf16: torch.Tensor, group: int, k8: torch.Tensor, scale: torch.Tensor,
                            stream=None) -> None:
    dim = k_bf16.shape[-1]
    _check(load().dsa_quantize_index_keys(_ptr(k_bf16), k_bf16.numel() // dim, dim, group, _ptr(k8), _ptr(scale),
                                          _stream(stream)))


def dsa_quantize_mxfp8(x_bf16: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
    dim = x_bf16.shape[-1]
    _check(load().dsa_quantize_mxfp8(_ptr(x_bf16), x_bf16.numel() // dim, dim, _ptr(codes), _ptr(scales),
                                     _stream(stream)))


def dsa_kv_fp8_row_bytes(d_latent: int, d_rope: int) -> int:
    return int(load().dsa_kv_fp8_row_bytes(d_latent, d_rope))


def dsa_quantize_kv(kv_bf16: torch.Tensor, d_latent: int, kv_fp8: torch.Tensor, stream=None) -> None:
    D = kv_bf16.shape[-1]
    _check(load().dsa_quantize_kv(_ptr(kv_bf16), kv_bf16.numel() // D, d_latent, D - d_latent, _ptr(kv_fp8),
                                  _stream(stream)))


def dsa_dequantize_index_keys(k8: torch.Tensor, scale: torch.Tensor, group: int, out: torch.Tensor,
                              stream=None) -> None:
    dim = k8.shape[-1]
    _check(load().dsa_dequantize_index_keys(_ptr(k8), _ptr(scale), k8.numel() // dim, dim, group, _ptr(out),
                                            _stream(stream)))


def dsa_read_device_status(stream=None) -> int:
    code = c_int32(0)
    _check(load().dsa_read_device_status(_stream(stream), ctypes.byref(code)))
    return int(code.value)


def dsa_debug_set_wait_limit(limit_ns: int) -> None:
    """Test hook: wall-time limit of the kernels' bounded waits (0 = default 2 s)."""
    _check(load().dsa_debug_set_wait_limit(int(limit_ns)))


def dsa_debug_withhold_signal(on: bool) -> None:
    """Test hook: the 128-head attention withholds its first P-ready signal."""
    _check(load().dsa_debug_withhold_signal(1 if on else 0))


def dsa_debug_delayed_copy(dst: torch.Tensor, src: torch.Tensor, delay_ns: int, stream=None) -> None:
    """Test hook: a kernel that lets dependent launches start at once, sleeps
    delay_ns, then copies src into dst (same byte size)."""
    nbytes = dst.numel() * dst.element_size()
    assert src.numel() * src.element_size() == nbytes
    _check(load().dsa_debug_delayed_copy(_ptr(dst), _ptr(src), nbytes, int(delay_ns), _stream(stream)))
