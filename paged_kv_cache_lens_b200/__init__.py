"""Paged KV-cache attention for B200 (sm_100a).

The compute path is the C-ABI library ``libpa.so`` (hand-written CUDA kernels),
reached through :mod:`paged_kv_cache_lens_b200.pa` (argument marshalling only).
:mod:`.workloads` draws seeded synthetic inputs; :mod:`.pool` sizes KV pools.
"""
