"""Indexed sparse attention (DSA) hot path for NVIDIA B200 (sm_100a).

Lightning Indexer scores -> per-row Top-K -> sparse MLA attention, as a C-ABI
CUDA library (``libdsa.so``) with a thin ctypes binding (:mod:`.binding`).
:mod:`.workloads` holds the seeded synthetic inputs.
"""
__all__ = ["workloads", "binding"]
