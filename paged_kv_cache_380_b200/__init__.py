"""Paged-KV-cache attention for B200 (sm_100a).

The work happens in ``libpagedkv.so`` (hand-written CUDA kernels behind a
C ABI, declared in ``include/pagedkv.h``).  ``paged_kv_cache_380_b200.ops``
is the thin ctypes binding with the same entry points
(``kv_cache_write``, ``paged_attention_decode``, ``paged_attention_prefill``);
``workloads`` holds the seeded synthetic inputs.  Importing the package does
not load the CUDA library; the first call into ``ops`` does, and fails loudly
if it is missing.
"""
__all__ = ["workloads"]
