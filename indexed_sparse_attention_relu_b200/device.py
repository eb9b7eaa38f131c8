"""Device copies of a seeded workload, ready for the C-ABI calls.

Marshalling only: the arrays of :mod:`.workloads` become torch tensors on a
CUDA device (bf16 bit patterns reinterpreted, int32 metadata copied). FP8
index keys are produced on the device by the library's own cache-write step
(``dsa_quantize_index_keys``), as in serving.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import binding as B
from .workloads import Workload, bf16_bits


def bf16_tensor(x: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(device)


@dataclasses.dataclass
class DeviceWorkload:
    wl: Workload
    batch: B.Batch
    q_idx: torch.Tensor
    w: torch.Tensor
    k_cache: torch.Tensor            # bf16 [B, L, dI] or uint8 codes
    k_scale: Optional[torch.Tensor]  # fp32 [B, L, dI/group] (FP8)
    k_bf16: Optional[torch.Tensor]   # bf16 keys (kept for the FP8 cache write)
    q: torch.Tensor
    kv: torch.Tensor
    q_mx: Optional[torch.Tensor] = None   # MXFP8 index inputs: E8M0 bytes of q_idx / k_cache
    k_mx: Optional[torch.Tensor] = None

    def indexer_in(self) -> B.dsa_indexer_in:
        if self.q_mx is not None:
            return B.indexer_in(self.q_idx, self.w, self.k_cache, q_mx=self.q_mx, k_mx=self.k_mx)
        return B.indexer_in(self.q_idx, self.w, self.k_cache, self.k_scale,
                            self.wl.scale_group if self.k_scale is not None else None)

    def mla_in(self) -> B.dsa_mla_in:
        return B.mla_in(self.q, self.kv, self.wl.dc, self.wl.softmax_scale)


def _cache_tensor(wl: Workload, tag: str, dev) -> torch.Tensor:
    """[B, Lmax, dim] bf16 cache; built sequence by sequence when the workload
    was made without host caches (rows past a sequence's length are zero)."""
    full = wl.k_idx if tag == "k_idx" else wl.kv
    if full is not None:
        return bf16_tensor(full, dev)
    dim = wl.dI if tag == "k_idx" else wl.D
    out = torch.zeros((wl.B, wl.Lmax, dim), dtype=torch.bfloat16, device=dev)
    for b in range(wl.B):
        n = int(wl.seq_lens[b])
        if n:
            out[b, :n] = bf16_tensor(wl.seq_rows(tag, b), dev)
    return out


def to_device(wl: Workload, device="cuda", keep_bf16_keys: bool = False) -> DeviceWorkload:
    dev = torch.device(device)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)
    batch = B.Batch(i32(wl.cu_q), i32(wl.q_pos), i32(wl.seq_lens), wl.Lmax)
    q_idx = bf16_tensor(wl.q_idx, dev)
    w = torch.from_numpy(np.ascontiguousarray(wl.w, np.float32)).to(dev)
    k_bf16 = _cache_tensor(wl, "k_idx", dev)
    k_scale = None
    k_cache = k_bf16
    if wl.key_dtype == "fp8":
        k_cache = torch.empty(k_bf16.shape, dtype=torch.uint8, device=dev)
        k_scale = torch.empty(k_bf16.shape[:-1] + (wl.dI // wl.scale_group,), dtype=torch.float32, device=dev)
        B.dsa_quantize_index_keys(k_bf16, wl.scale_group, k_cache, k_scale)
        if not keep_bf16_keys:
            k_bf16 = None
    q = bf16_tensor(wl.q, dev)
    kv = _cache_tensor(wl, "kv", dev)
    return DeviceWorkload(wl, batch, q_idx, w, k_cache, k_scale, k_bf16 if wl.key_dtype == "fp8" else None, q, kv)


def subset(dw: DeviceWorkload, rows) -> DeviceWorkload:
    """The same caches with only the query tokens ``rows`` (sorted) kept."""
    wl = dw.wl
    rows = np.asarray(rows, np.int64)
    b = wl.seq_of_token()[rows]
    counts = np.bincount(b, minlength=wl.B)
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    dev = dw.q.device
    r = torch.from_numpy(rows).to(dev)
    sub_wl = dataclasses.replace(wl, T=len(rows), cu_q=cu, q_pos=wl.q_pos[rows].copy(), q_idx=wl.q_idx[rows],
                                 w=wl.w[rows], q=wl.q[rows])
    batch = B.Batch(torch.from_numpy(cu).to(dev), dw.batch.q_pos[r].contiguous(), dw.batch.seq_lens, wl.Lmax)
    return dataclasses.replace(dw, wl=sub_wl, batch=batch, q_idx=dw.q_idx[r].contiguous(), w=dw.w[r].contiguous(),
                               q=dw.q[r].contiguous())


def to_paged(dw: DeviceWorkload, page_size: int, seed: int = 0, spare_pages: int = 3,
             fill: float = 1000.0) -> DeviceWorkload:
    """The same workload with every cache moved into one page pool.

    Page placement comes from :func:`.workloads.page_layout`; rows are copied
    page by page (layout only). Pool rows no sequence owns hold ``fill`` (FP8
    index-key codes: 0x7E, scales: 1; packed FP8 KV rows: bytes 0x11), so a
    kernel that read a wrong row would show it.
    """
    from . import workloads as W
    wl = dw.wl
    table, num_pages = W.page_layout(wl.seq_lens, wl.Lmax, page_size, seed, spare_pages)
    rows = num_pages * page_size
    src = np.full(rows, -1, np.int64)
    for b in range(wl.B):
        for j in np.nonzero(table[b] >= 0)[0]:
            n = min(page_size, wl.Lmax - int(j) * page_size)
            pg = int(table[b, j])
            src[pg * page_size:pg * page_size + n] = b * wl.Lmax + int(j) * page_size + np.arange(n)
    dev = dw.q.device
    src_t = torch.from_numpy(src).to(dev)
    have = src_t >= 0

    def scatter(cache: torch.Tensor, fill_value) -> torch.Tensor:
        flat = cache.reshape(wl.B * wl.Lmax, -1)
        pool = torch.full((rows, flat.shape[1]), fill_value, dtype=cache.dtype, device=dev)
        pool[have] = flat[src_t[have]]
        return pool

    fp8 = dw.k_scale is not None or dw.k_mx is not None
    k_cache = scatter(dw.k_cache, 0x7E if fp8 else fill)
    k_scale = scatter(dw.k_scale, 1.0) if dw.k_scale is not None else None
    k_mx = scatter(dw.k_mx, 127) if dw.k_mx is not None else None   # E8M0 127 = 2^0
    kv = scatter(dw.kv, 0x11 if dw.kv.dtype == torch.uint8 else fill)  # packed FP8 rows: finite filler
    batch = B.Batch(dw.batch.cu_q, dw.batch.q_pos, dw.batch.seq_lens, wl.Lmax,
                    block_table=torch.from_numpy(table).to(dev), page_size=page_size, num_pages=num_pages)
    return dataclasses.replace(dw, batch=batch, k_cache=k_cache, k_scale=k_scale, kv=kv, k_bf16=None, k_mx=k_mx)


def with_fp8_kv(dw: DeviceWorkload) -> DeviceWorkload:
    """The same workload with its latent KV cache written as packed FP8 rows
    by the library's own cache-write step (dsa_quantize_kv), as in serving."""
    wl = dw.wl
    rows = dw.kv.reshape(-1, wl.D)
    kv8 = torch.empty((rows.shape[0], B.dsa_kv_fp8_row_bytes(wl.dc, wl.dr)), dtype=torch.uint8, device=dw.kv.device)
    B.dsa_quantize_kv(rows, wl.dc, kv8)
    return dataclasses.replace(dw, kv=kv8.reshape(dw.kv.shape[:-1] + (kv8.shape[-1],)))


def with_mxfp8_index(dw: DeviceWorkload) -> DeviceWorkload:
    """The same workload with MXFP8 index queries and keys (group 32, E8M0
    scales), written by the library's dsa_quantize_mxfp8 from the bf16 ones."""
    wl = dw.wl
    dev = dw.q.device
    keys = dw.k_bf16 if dw.k_bf16 is not None else dw.k_cache
    assert keys.dtype == torch.bfloat16, "MXFP8 index inputs are made from bf16 keys"
    k8 = torch.empty(keys.shape, dtype=torch.uint8, device=dev)
    kmx = torch.empty(keys.shape[:-1] + (wl.dI // 32,), dtype=torch.uint8, device=dev)
    B.dsa_quantize_mxfp8(keys, k8, kmx)
    q8 = torch.empty(dw.q_idx.shape, dtype=torch.uint8, device=dev)
    qmx = torch.empty(dw.q_idx.shape[:-1] + (wl.dI // 32,), dtype=torch.uint8, device=dev)
    B.dsa_quantize_mxfp8(dw.q_idx, q8, qmx)
    return dataclasses.replace(dw, q_idx=q8, k_cache=k8, k_scale=None, k_bf16=None, q_mx=qmx, k_mx=kmx)
