"""Shared test helpers: pools filled from a Workload by the ORACLE's cache write."""
import numpy as np

from paged_kv_cache_lens_b200 import workloads as wl

# a NaN in each pool format, so a read of a never-written slot poisons the result
NAN_FILL = {wl.BF16: 0x7FC0, wl.F16: 0x7E00, wl.FP8_E4M3: 0x7F}


def empty_pool(W, fill=None):
    shape = (W.num_blocks, W.num_kv_heads, W.block_size, W.head_dim)
    dt = np.uint8 if W.kv_dtype == wl.FP8_E4M3 else np.uint16
    f = NAN_FILL[W.kv_dtype] if fill is None else fill
    return np.full(shape, f, dt), np.full(shape, f, dt)


def oracle_pools(oracle, W, include_new=True):
    """Pool contents after the cached context (and the step's new tokens) are
    written by the oracle's cache write."""
    kc, vc = empty_pool(W)
    if len(W.prefill_slots):
        oracle.reshape_and_cache(W.prefill_k, W.prefill_v, W.src_dtype, W.prefill_slots, kc, vc,
                                 W.block_size, W.kv_dtype, W.k_scale, W.v_scale)
    if include_new and len(W.new_slots):
        oracle.reshape_and_cache(W.new_k, W.new_v, W.src_dtype, W.new_slots, kc, vc,
                                 W.block_size, W.kv_dtype, W.k_scale, W.v_scale)
    return kc, vc


def oracle_attention(oracle, W, kc, vc, **kw):
    return oracle.paged_attention(W.q, W.q_dtype, W.cu_seqlens_q, W.seqlens_k, kc, vc,
                                  W.kv_dtype, W.block_tables, W.scale, W.k_scale, W.v_scale, **kw)
