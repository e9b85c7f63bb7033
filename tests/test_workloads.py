"""Host-side checks of the seeded input generator and the pool arithmetic."""
import json
import os

import numpy as np
import pytest

from paged_kv_cache_lens_b200 import pool
from paged_kv_cache_lens_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _check_structure(W):
    bs = W.block_size
    assert W.block_tables.dtype == np.int32 and W.seqlens_k.dtype == np.int32
    assert W.cu_seqlens_q[0] == 0 and np.all(np.diff(W.cu_seqlens_q) >= 0)
    for r in range(W.num_seqs):
        n = -(-int(W.seqlens_k[r]) // bs)
        row = W.block_tables[r]
        assert np.all((row[:n] >= 0) & (row[:n] < W.num_blocks))
        assert np.all(row[n:] == -1)
    # every written slot is unique within the prefill and within the step
    for slots in (W.prefill_slots, W.new_slots[W.new_slots >= 0]):
        assert len(np.unique(slots)) == len(slots)
        assert np.all(slots < W.num_blocks * bs)
    allw = np.concatenate([W.prefill_slots, W.new_slots[W.new_slots >= 0]])
    assert len(np.unique(allw)) == len(allw)


@pytest.mark.parametrize("i", [1, 2, 3, 4, 5])
def test_reference_configs_small_batch(i):
    W = wl.config(i, batch=None if i == 1 else 6)
    _check_structure(W)
    assert W.decode == (i != 4)


def test_config1_exact_shape():
    W = wl.config(1)
    assert list(W.seqlens_k) == [1, 17, 40, 100]
    assert W.num_blocks == 64 and W.num_q_heads == W.num_kv_heads == 2 and W.head_dim == 64
    assert W.q_dtype == wl.F16 and W.kv_dtype == wl.F16
    used = [b for r in range(4) for b in W.block_tables[r] if b >= 0]
    assert len(used) == 1 + 2 + 3 + 7 == len(set(used))
    assert W.scale == np.float32(1 / 8)


def test_config4_mixed_step_shape():
    W = wl.config(4, batch=10)
    q_lens = W.q_lens
    assert np.all(q_lens[:10] == 1) and np.all(q_lens[10:] == 512)
    assert list(W.seqlens_k[10:]) == [512, 1536, 2560, 3584]
    assert W.total_q == 10 + 4 * 512 and W.num_q_heads == 32 and W.num_kv_heads == 8


def test_config5_shared_prefix():
    W = wl.config(5, batch=8)
    assert np.all(W.block_tables[:, :128] == W.block_tables[0, :128])
    assert len(np.unique(W.block_tables[0, :128])) == 128
    assert W.kv_dtype == wl.FP8_E4M3 and W.k_scale.shape == (8,)
    # scales leave every value within the finite range
    kf = np.abs(wl.bits_to_f32(W.prefill_k, wl.BF16)).max(axis=(0, 2))
    assert np.all(kf / W.k_scale <= np.float32(448.0) * (1 + 1e-6))
    private = W.block_tables[:, 128:]
    ids = private[private >= 0]
    assert len(np.unique(ids)) == len(ids) and not set(ids) & set(W.block_tables[0, :128])


def test_determinism():
    a, b = wl.config(3, batch=5), wl.config(3, batch=5)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.block_tables, b.block_tables)
    assert np.array_equal(a.prefill_k, b.prefill_k)
    c = wl.config(3, seed=77, batch=5)
    assert not np.array_equal(a.q, c.q)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-39], np.float32)
    bits = wl.f32_to_bf16_bits(x)
    # 1 + 2^-8 is half way between 1 and 1 + 2^-7: ties to even (1.0)
    assert list(bits[:2]) == [0x3F80, 0x3F80]
    assert bits[2] == 0x3F82              # 1 + 3*2^-8 -> 1 + 2^-6 (even)
    assert bits[3] == 0xC020


def test_pool_sizing_examples():
    g = json.load(open(os.path.join(GOLDEN, "kv_sizing.json")))
    pb = g["per_block"]
    assert pool.kv_bytes_per_block(pb["block_size"], pb["num_layers"], pb["num_kv_heads"],
                                   pb["head_dim"], pb["dtype_bytes"]) == pb["bytes"]
    mc = g["max_concurrency"]
    assert pool.kv_bytes_per_token(mc["num_layers"], mc["num_kv_heads"], mc["head_dim"],
                                   mc["dtype_bytes"]) == mc["bytes_per_token"]
    assert pool.max_concurrent_sequences(mc["kv_budget_bytes"], mc["avg_context"], mc["num_layers"],
                                         mc["num_kv_heads"], mc["head_dim"], mc["dtype_bytes"],
                                         mc["block_size"]) == mc["sequences"]
    bk = g["batch_kv_bytes"]
    assert bk["batch"] * bk["seq"] * pool.kv_bytes_per_token(
        bk["num_layers"], bk["num_kv_heads"], bk["head_dim"], bk["dtype_bytes"]) == bk["bytes"]
