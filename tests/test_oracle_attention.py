"""Pins for the oracle's attention over the paged cache (CPU only).

Paging changes only where K/V live, never the result ("PagedAttention 与
Continuous Batching", §3.6 PagedAttention Kernel; §10.8 FAQ: a prefix-cache hit
equals recomputation up to rounding).  Each test below ties the oracle to
something other than itself: a closed form, a special case, brute force on
tiny inputs, PyTorch's float64 scaled-dot-product attention, or the
independent NumPy twin.
"""
import math

import numpy as np
import pytest
import torch

from oracle import pa_oracle_np as npo
from paged_kv_cache_lens_b200 import workloads as wl
from tests._helpers import NAN_FILL, oracle_attention, oracle_pools


def _f64(bits, dtype):
    return npo.to_f64(bits, dtype)


def _contiguous_kv(W, kc, vc, r):
    """[kv_len, Hkv, D] float64 K/V of request r, gathered by hand."""
    L = int(W.seqlens_k[r])
    t = np.arange(L)
    blk = W.block_tables[r, t // W.block_size]
    k = _f64(kc[blk, :, t % W.block_size, :], W.kv_dtype)
    v = _f64(vc[blk, :, t % W.block_size, :], W.kv_dtype)
    if W.kv_dtype == wl.FP8_E4M3:
        k = k * W.k_scale.astype(np.float64)[None, :, None]
        v = v * W.v_scale.astype(np.float64)[None, :, None]
    return k, v


def _sdpa_reference(W, kc, vc):
    """torch float64 SDPA with an explicit bottom-right causal mask."""
    out = np.zeros((W.total_q, W.num_q_heads, W.head_dim))
    g = W.num_q_heads // W.num_kv_heads
    q = _f64(W.q, W.q_dtype)
    for r in range(W.num_seqs):
        r0, r1 = int(W.cu_seqlens_q[r]), int(W.cu_seqlens_q[r + 1])
        L = int(W.seqlens_k[r])
        if L == 0 or r1 == r0:
            continue
        k, v = _contiguous_kv(W, kc, vc, r)
        kt = torch.from_numpy(k).transpose(0, 1).repeat_interleave(g, 0)   # [Hq, L, D]
        vt = torch.from_numpy(v).transpose(0, 1).repeat_interleave(g, 0)
        qt = torch.from_numpy(q[r0:r1]).transpose(0, 1)                    # [Hq, qn, D]
        qn = r1 - r0
        rows = torch.arange(qn)[:, None]
        cols = torch.arange(L)[None, :]
        mask = cols <= (L - qn + rows)
        o = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=mask, scale=float(W.scale))
        out[r0:r1] = o.transpose(0, 1).numpy()
    return out


def _small_varlen(seed=21, dtype=wl.BF16, kv_dtype=None, hq=4, hkv=2, d=32):
    q_lens = [1, 1, 5, 17, 1, 33, 3]
    kv_lens = [1, 40, 5, 50, 16, 33, 70]
    return wl.build_workload("small", seed, q_lens, kv_lens, hq, hkv, d, dtype=dtype,
                             kv_dtype=kv_dtype)


def test_single_key_returns_its_value_exactly(oracle):
    W = wl.build_workload("one", 1, [1, 1], [1, 1], 4, 2, 16)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    for r in range(2):
        v = _f64(W.new_v[r], W.src_dtype)            # [Hkv, D]
        for hq in range(4):
            assert np.array_equal(out[r, hq], v[hq // 2])


def test_uniform_keys_give_mean_of_values(oracle):
    W = wl.build_workload("uni", 2, [1, 1, 1], [37, 5, 100], 2, 1, 8)
    W.prefill_k[:] = W.prefill_k[0]
    W.new_k[:] = W.prefill_k[0]
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    for r in range(3):
        _, v = _contiguous_kv(W, kc, vc, r)
        np.testing.assert_allclose(out[r, 0], v[:, 0].mean(axis=0), rtol=0, atol=1e-14)


def test_hand_case_two_keys():
    """D = 1, q = 1, keys {0, 1}, scale = fp32(ln 2), values {0, 3}:
    weights 1/(1+e^s), e^s/(1+e^s) with s = fp32(ln 2), so out = 3e^s/(1+e^s) ~ 2."""
    from oracle import pa_oracle as oracle
    bs = 16
    kc = np.zeros((1, 1, bs, 1), np.uint16)
    vc = np.zeros((1, 1, bs, 1), np.uint16)
    kc[0, 0, 1, 0] = 0x3F80            # bf16 1.0
    vc[0, 0, 1, 0] = 0x4040            # bf16 3.0
    q = np.array([[[0x3F80]]], np.uint16)
    s = float(np.float32(math.log(2.0)))
    out = oracle.paged_decode(q, wl.BF16, np.array([2], np.int32), kc, vc, wl.BF16,
                              np.array([[0]], np.int32), s)
    want = 3 * math.exp(s) / (1 + math.exp(s))
    assert abs(out[0, 0, 0] - want) < 1e-15
    assert abs(out[0, 0, 0] - 2.0) < 1e-7


def test_zero_context_gives_zeros(oracle):
    W = wl.build_workload("z", 3, [1, 1], [3, 2], 2, 2, 8)
    W.seqlens_k[0] = 0
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    assert np.all(out[0] == 0.0) and np.all(np.isfinite(out[1]))


def test_matches_torch_sdpa_float64_and_numpy_twin(oracle):
    for kv_dtype, dtype in [(None, wl.BF16), (None, wl.F16), (wl.FP8_E4M3, wl.BF16)]:
        W = _small_varlen(dtype=dtype, kv_dtype=kv_dtype)
        kc, vc = oracle_pools(oracle, W)
        out = oracle_attention(oracle, W, kc, vc)
        ref = _sdpa_reference(W, kc, vc)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
        tw = npo.paged_attention(W.q, W.q_dtype, W.cu_seqlens_q, W.seqlens_k, kc, vc, W.kv_dtype,
                                 W.block_tables, W.scale, W.k_scale, W.v_scale)
        np.testing.assert_allclose(out, tw, rtol=0, atol=1e-12)


def test_invariant_under_physical_block_permutation(oracle):
    W = _small_varlen(seed=22)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    perm = np.random.default_rng(9).permutation(W.num_blocks)    # new id of old block b
    kp, vp = np.empty_like(kc), np.empty_like(vc)
    kp[perm], vp[perm] = kc, vc
    bt = W.block_tables.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    W2 = W
    old = W.block_tables
    W2.block_tables = bt
    out2 = oracle_attention(oracle, W2, kp, vp)
    W.block_tables = old
    assert np.array_equal(out, out2)


def test_shared_prefix_equals_unshared_copies(oracle):
    """Sequences whose first blocks are the same physical blocks give the
    same result, bit for bit, as copies of that prefix in private blocks."""
    W = wl.build_workload("sp", 23, [1, 1, 1], [64, 80, 33], 4, 2, 16, kv_dtype=wl.FP8_E4M3,
                          shared_prefix_len=32)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    # give requests 1 and 2 private copies of the two shared blocks
    nb = W.num_blocks
    kc2 = np.concatenate([kc, np.zeros((4,) + kc.shape[1:], kc.dtype)])
    vc2 = np.concatenate([vc, np.zeros((4,) + vc.shape[1:], vc.dtype)])
    bt = W.block_tables.copy()
    for j, r in enumerate([1, 2]):
        for i in range(2):
            src = bt[r, i]
            dst = nb + 2 * j + i
            kc2[dst], vc2[dst] = kc[src], vc[src]
            bt[r, i] = dst
    assert bt[1, 0] != bt[0, 0]
    old = W.block_tables
    W.block_tables, W.num_blocks = bt, nb + 4
    out2 = oracle_attention(oracle, W, kc2, vc2)
    W.block_tables, W.num_blocks = old, nb
    assert np.array_equal(out, out2)


def test_brute_force_tiny_all_splits(oracle):
    """D <= 4, L <= 40, every split of L into cached + new rows, against a
    direct softmax written out with Python floats."""
    rng = np.random.default_rng(24)
    for L in [1, 2, 7, 16, 17, 40]:
        splits = range(1, L + 1) if L <= 17 else (1, 2, 20, 39, 40)
        for q_len in splits:
            for d in (1, 3, 4):
                W = wl.build_workload("bf", int(rng.integers(1 << 30)), [q_len], [L], 2, 1, d,
                                      dtype=wl.F16)
                kc, vc = oracle_pools(oracle, W)
                out = oracle_attention(oracle, W, kc, vc)
                k, v = _contiguous_kv(W, kc, vc, 0)
                q = _f64(W.q, W.q_dtype)
                for i in range(q_len):
                    for h in range(2):
                        n = L - q_len + i + 1
                        s = [W.scale * sum(q[i, h, x] * k[t, 0, x] for x in range(d))
                             for t in range(n)]
                        m = max(s)
                        w = [math.exp(z - m) for z in s]
                        den = sum(w)
                        for x in range(d):
                            want = sum(w[t] * v[t, 0, x] for t in range(n)) / den
                            assert abs(out[i, h, x] - want) < 1e-12


def test_lse_merge_of_partitions_equals_one_pass(oracle):
    """Split the keys of a sequence into 16-aligned partitions; attention over
    each partition plus the log-sum-exp merge M = max lse_p, out = sum_p
    e^(lse_p - M) out_p / sum_p e^(lse_p - M) reproduces the one-pass result."""
    W = wl.build_workload("lse", 25, [1], [300], 4, 2, 32)
    kc, vc = oracle_pools(oracle, W)
    full, lse_full = oracle_attention(oracle, W, kc, vc, with_lse=True)
    for bounds in ([0, 128, 256, 300], [0, 16, 300], [0, 288, 300]):
        outs, lses = [], []
        for a, b in zip(bounds, bounds[1:]):
            table = W.block_tables[:, a // 16:]
            o, l = oracle.paged_attention(
                W.q, W.q_dtype, np.array([0, 1], np.int32), np.array([b - a], np.int32), kc, vc,
                W.kv_dtype, np.ascontiguousarray(table), W.scale, with_lse=True)
            outs.append(o[0])
            lses.append(l[0])
        lses = np.array(lses)                              # [P, Hq]
        M = lses.max(axis=0)
        w = np.exp(lses - M)
        merged = (w[:, :, None] * np.array(outs)).sum(0) / w.sum(0)[:, None]
        np.testing.assert_allclose(merged, full[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(M + np.log(w.sum(0)), lse_full[0], rtol=0, atol=1e-12)


def test_chunk_row_equals_decode_with_shorter_context(oracle):
    """Row i of a chunk (q_len rows over kv_len keys) equals a decode whose
    context is kv_len - q_len + i + 1 keys of the same table."""
    W = wl.build_workload("vc", 26, [1, 20], [9, 45], 4, 2, 16)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    for i in range(20):
        L = 45 - 20 + i + 1
        o = oracle.paged_decode(W.q[1 + i:2 + i], W.q_dtype, np.array([L], np.int32), kc, vc,
                                W.kv_dtype, W.block_tables[1:2], W.scale)
        assert np.array_equal(o[0], out[1 + i])


def test_chunk_without_cache_is_causal_self_attention(oracle):
    """A request whose q_len equals kv_len is ordinary causal self-attention
    (top-left and bottom-right alignment coincide for a square mask)."""
    W = wl.build_workload("cs", 27, [37], [37], 2, 2, 16)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    k, v = _contiguous_kv(W, kc, vc, 0)
    q = torch.from_numpy(_f64(W.q, W.q_dtype)).transpose(0, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, torch.from_numpy(k).transpose(0, 1), torch.from_numpy(v).transpose(0, 1),
        is_causal=True, scale=float(W.scale)).transpose(0, 1).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_gqa_groups_are_contiguous(oracle):
    """Query head hq reads KV head hq // (Hq / Hkv)."""
    W = wl.build_workload("g", 28, [1], [20], 8, 2, 8)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    vc2 = vc.copy()
    vc2[:, 1] = vc[:, 1] ^ np.uint16(0x8000)             # negate every value of KV head 1
    out2 = oracle_attention(oracle, W, kc, vc2)
    assert np.array_equal(out[0, :4], out2[0, :4])
    np.testing.assert_array_equal(out[0, 4:], -out2[0, 4:])


def test_pairs_mode_matches_full(oracle):
    W = _small_varlen(seed=29)
    kc, vc = oracle_pools(oracle, W)
    full = oracle_attention(oracle, W, kc, vc, num_threads=3)
    rows = np.array([0, 5, 6, 40, W.total_q - 1])
    heads = np.array([0, 3, 1, 2, 3])
    part = oracle_attention(oracle, W, kc, vc, pairs=(rows, heads))
    for j in range(len(rows)):
        assert np.array_equal(part[j], full[rows[j], heads[j]])


def test_never_reads_unwritten_slots(oracle):
    """Pools start as NaN; every config-1 output is finite, so only written
    slots below each context length were read."""
    W = wl.config(1)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc)
    assert np.all(np.isfinite(out))
    assert np.isnan(_f64(kc, W.kv_dtype)).any()


def _relayout(W, kc, vc, bs, seed):
    """The same logical K/V of every request, moved byte for byte into a pool
    of `bs`-token blocks under a fresh seeded random block table (the paging
    of "PagedAttention 与 Continuous Batching", §3.3: token t of a request
    lives at table[t / bs] * bs + t % bs, for any block size of §3.7)."""
    import dataclasses
    rng = np.random.default_rng(seed)
    need = [-(-int(L) // bs) for L in W.seqlens_k]
    nb = max(1, sum(need) + 3)
    ids = rng.permutation(nb).astype(np.int32)
    tables = np.full((W.num_seqs, max(need) + 1), -1, np.int32)
    shape = (nb, W.num_kv_heads, bs, W.head_dim)
    k2, v2 = np.zeros(shape, kc.dtype), np.zeros(shape, vc.dtype)
    cur = 0
    for r, n in enumerate(need):
        tables[r, :n] = ids[cur:cur + n]
        cur += n
        t = np.arange(int(W.seqlens_k[r]))
        old_b, old_o = W.block_tables[r, t // W.block_size], t % W.block_size
        new_b, new_o = tables[r, t // bs], t % bs
        k2[new_b, :, new_o, :] = kc[old_b, :, old_o, :]
        v2[new_b, :, new_o, :] = vc[old_b, :, old_o, :]
    W2 = dataclasses.replace(W, block_size=bs, block_tables=tables, num_blocks=nb)
    return W2, k2, v2


@pytest.mark.parametrize("kv", [None, wl.FP8_E4M3])
@pytest.mark.parametrize("bs", [8, 32])
def test_block_size_changes_nothing(oracle, bs, kv):
    """The same logical cache laid out in 8- or 32-token blocks gives bitwise
    the result of 16-token blocks, and matches float64 SDPA."""
    W = _small_varlen(seed=41, kv_dtype=kv)
    kc, vc = oracle_pools(oracle, W)
    want = oracle_attention(oracle, W, kc, vc)
    W2, k2, v2 = _relayout(W, kc, vc, bs, seed=42)
    got = oracle_attention(oracle, W2, k2, v2)
    assert np.array_equal(got, want)
    np.testing.assert_allclose(got, _sdpa_reference(W2, k2, v2), rtol=0, atol=1e-12)


@pytest.mark.parametrize("kv", [None, wl.FP8_E4M3])
@pytest.mark.parametrize("bs", [8, 32])
def test_cache_write_at_other_block_sizes_matches_numpy_twin(oracle, bs, kv):
    W = wl.build_workload("bsw", 43, [1, 9, 1, 3], [20, 9, 70, 41], 4, 2, 16, kv_dtype=kv,
                          block_size=bs)
    kc, vc = oracle_pools(oracle, W)
    kt = np.full_like(kc, NAN_FILL[W.kv_dtype])                 # the oracle pools' fill too
    vt = np.full_like(vc, NAN_FILL[W.kv_dtype])
    for k, v, s in ((W.prefill_k, W.prefill_v, W.prefill_slots), (W.new_k, W.new_v, W.new_slots)):
        npo.reshape_and_cache(k, v, W.src_dtype, s, kt, vt, W.kv_dtype, W.k_scale, W.v_scale)
    assert np.array_equal(kt, kc) and np.array_equal(vt, vc)
