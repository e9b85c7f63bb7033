"""Pins for the oracle's cache write and block addressing (CPU only).

"PagedAttention 与 Continuous Batching", §3.3 (数据结构): a token at logical
position t lives in logical block t // 16 at offset t % 16, and the block
table maps logical to physical blocks; §2.5 step 4 hands the per-token
physical slot to the forward pass as slot_mapping.
"""
import json
import os

import numpy as np
import pytest

from oracle import pa_oracle_np as npo
from paged_kv_cache_lens_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pool(nb, hkv, bs, d, fill, dtype=np.uint16):
    return np.full((nb, hkv, bs, d), fill, dtype=dtype)


def test_token18_example_lands_in_block42_offset2(oracle):
    g = json.load(open(os.path.join(GOLDEN, "paging_examples.json")))
    ex, bs = g["sequence_a"], g["block_size"]
    table = np.array(ex["block_table"], np.int64)
    t = ex["token"]
    assert t // bs == ex["logical_block"] and t % bs == ex["offset"]
    assert table[t // bs] == ex["physical_block"]
    slot = int(table[t // bs]) * bs + t % bs
    assert slot == ex["slot"]
    # the oracle writes that token exactly there and nowhere else
    hkv, d = 2, 8
    k = np.arange(hkv * d, dtype=np.uint16).reshape(1, hkv, d) + 1
    v = k + 100
    kc, vc = _pool(64, hkv, bs, d, 0xFFFF), _pool(64, hkv, bs, d, 0xFFFF)
    oracle.reshape_and_cache(k, v, wl.BF16, np.array([slot]), kc, vc, bs, wl.BF16)
    assert np.array_equal(kc[42, :, 2, :], k[0]) and np.array_equal(vc[42, :, 2, :], v[0])
    mask = np.ones(kc.shape, bool)
    mask[42, :, 2, :] = False
    assert np.all(kc[mask] == 0xFFFF) and np.all(vc[mask] == 0xFFFF)


def test_seq33_uses_three_blocks_and_never_the_fourth(oracle):
    """A 33-token sequence reads ceil(33/16) = 3 table entries; a fourth
    entry of -1 (the page's '?') is never dereferenced."""
    g = json.load(open(os.path.join(GOLDEN, "paging_examples.json")))["sequence_b"]
    bs = 16
    n = g["num_tokens"]
    assert -(-n // bs) == g["blocks_used"]
    table = np.array([g["block_table"]], np.int32)
    assert table[0, (n - 1) // bs] == g["last_token_physical_block"]
    assert (n - 1) % bs == g["last_token_offset"]
    hkv, d = 1, 4
    kc = np.full((32, hkv, bs, d), 0x3F80, np.uint16)     # bf16 1.0 everywhere
    vc = np.full((32, hkv, bs, d), 0x3F80, np.uint16)
    q = np.full((1, 1, d), 0x3F80, np.uint16)
    out = oracle.paged_decode(q, wl.BF16, np.array([n], np.int32), kc, vc, wl.BF16, table, 0.5)
    assert np.all(out == 1.0)
    with pytest.raises(ValueError):   # the same table with a 49-token context reads -1
        oracle.paged_decode(q, wl.BF16, np.array([49], np.int32), kc, vc, wl.BF16, table, 0.5)


@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_scatter_roundtrip_and_sentinel(oracle, dtype):
    rng = np.random.default_rng(11)
    nb, hkv, bs, d, T = 40, 3, 16, 24, 300
    slots = rng.choice(nb * bs, T, replace=False).astype(np.int64)
    slots[rng.choice(T, 20, replace=False)] = -1                     # padding tokens
    k = wl.randn_bits(rng, (T, hkv, d), dtype)
    v = wl.randn_bits(rng, (T, hkv, d), dtype)
    kc, vc = _pool(nb, hkv, bs, d, 0xFFFF), _pool(nb, hkv, bs, d, 0xFFFF)
    oracle.reshape_and_cache(k, v, dtype, slots, kc, vc, bs, dtype)
    written = np.zeros((nb, bs), bool)
    for i, s in enumerate(slots.tolist()):
        if s < 0:
            continue
        written[s // bs, s % bs] = True
        assert np.array_equal(kc[s // bs, :, s % bs, :], k[i])        # gather = input
        assert np.array_equal(vc[s // bs, :, s % bs, :], v[i])
    untouched = ~written[:, None, :, None].repeat(hkv, 1).repeat(d, 3)
    assert np.all(kc[untouched] == 0xFFFF) and np.all(vc[untouched] == 0xFFFF)
    # twin agrees bit for bit
    kt, vt = _pool(nb, hkv, bs, d, 0xFFFF), _pool(nb, hkv, bs, d, 0xFFFF)
    npo.reshape_and_cache(k, v, dtype, slots, kt, vt, dtype)
    assert np.array_equal(kt, kc) and np.array_equal(vt, vc)


def test_scatter_token_stride(oracle):
    """Rows inside a fused QKV buffer: token i starts at i * token_stride."""
    rng = np.random.default_rng(12)
    T, hq, hkv, d, bs = 9, 4, 2, 8, 16
    qkv = wl.randn_bits(rng, (T, (hq + 2 * hkv) * d), wl.BF16)
    k = qkv[:, hq * d:]
    v = qkv[:, (hq + hkv) * d:]
    slots = np.arange(T, dtype=np.int64) * 3
    kc, vc = _pool(8, hkv, bs, d, 0), _pool(8, hkv, bs, d, 0)
    oracle.reshape_and_cache(k, v, wl.BF16, slots, kc, vc, bs, wl.BF16,
                             token_stride=(hq + 2 * hkv) * d)
    for i in range(T):
        s = int(slots[i])
        assert np.array_equal(kc[s // bs, :, s % bs, :].ravel(), qkv[i, hq * d:(hq + hkv) * d])
        assert np.array_equal(vc[s // bs, :, s % bs, :].ravel(), qkv[i, (hq + hkv) * d:])


def test_fp8_scatter_is_rne_of_fp32_quotient(oracle):
    rng = np.random.default_rng(13)
    nb, hkv, bs, d, T = 8, 2, 16, 32, 100
    slots = rng.choice(nb * bs, T, replace=False).astype(np.int64)
    k = wl.randn_bits(rng, (T, hkv, d), wl.BF16)
    v = wl.randn_bits(rng, (T, hkv, d), wl.BF16)
    ks = np.array([0.01, 0.0071], np.float32)     # some values saturate at 448
    vs = np.array([0.003, 0.02], np.float32)
    kc, vc = _pool(nb, hkv, bs, d, 0x7F, np.uint8), _pool(nb, hkv, bs, d, 0x7F, np.uint8)
    oracle.reshape_and_cache(k, v, wl.BF16, slots, kc, vc, bs, wl.FP8_E4M3, ks, vs)
    kf, vf = wl.bits_to_f32(k, wl.BF16), wl.bits_to_f32(v, wl.BF16)
    for i in range(0, T, 7):
        s = int(slots[i])
        for h in range(hkv):
            for dd in range(0, d, 5):
                assert kc[s // bs, h, s % bs, dd] == oracle.e4m3_from_float(
                    float(np.float32(kf[i, h, dd]) / ks[h]))
                assert vc[s // bs, h, s % bs, dd] == oracle.e4m3_from_float(
                    float(np.float32(vf[i, h, dd]) / vs[h]))
    assert np.any(kc == 0x7E) or np.any(kc == 0xFE)               # saturation exercised
    kt, vt = _pool(nb, hkv, bs, d, 0x7F, np.uint8), _pool(nb, hkv, bs, d, 0x7F, np.uint8)
    npo.reshape_and_cache(k, v, wl.BF16, slots, kt, vt, wl.FP8_E4M3, ks, vs)
    assert np.array_equal(kt, kc) and np.array_equal(vt, vc)


def test_scatter_rejects_slot_outside_pool(oracle):
    k = np.zeros((1, 1, 4), np.uint16)
    kc = _pool(2, 1, 16, 4, 0)
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(k, k, wl.BF16, np.array([32]), kc, kc.copy(), 16, wl.BF16)
