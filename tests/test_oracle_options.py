"""Pins for the oracle's sliding-window and ALiBi options (CPU only).

"PagedAttention 与 Continuous Batching", §10.8 (FAQ) lists sliding window and
ALiBi among the variants paged kernels must cover.  Readings: with a window
of W a query at position p sees keys p-W+1 .. p; ALiBi adds slope_h * (t - p)
to the scaled logit of key t for query head h.
"""
import math

import numpy as np
import pytest
import torch

from oracle import pa_oracle_np as npo
from paged_kv_cache_lens_b200 import workloads as wl
from tests._helpers import oracle_attention, oracle_pools


def _reference(W, kc, vc, window=0, slopes=None):
    """float64 SDPA with an explicit additive bias (mask and ALiBi)."""
    g = W.num_q_heads // W.num_kv_heads
    out = np.zeros((W.total_q, W.num_q_heads, W.head_dim))
    q = npo.to_f64(W.q, W.q_dtype)
    for r in range(W.num_seqs):
        r0, r1, L = int(W.cu_seqlens_q[r]), int(W.cu_seqlens_q[r + 1]), int(W.seqlens_k[r])
        if L == 0 or r1 == r0:
            continue
        t = np.arange(L)
        blk = W.block_tables[r, t // W.block_size]
        k = npo.to_f64(kc[blk, :, t % W.block_size, :], W.kv_dtype)
        v = npo.to_f64(vc[blk, :, t % W.block_size, :], W.kv_dtype)
        pos = L - (r1 - r0) + np.arange(r1 - r0)
        vis = t[None, :] <= pos[:, None]
        if window > 0:
            vis &= t[None, :] >= pos[:, None] - window + 1
        bias = np.where(vis, 0.0, -np.inf)[None].repeat(W.num_q_heads, 0)     # [H, q, L]
        if slopes is not None:
            bias = bias + np.asarray(slopes, np.float32).astype(np.float64)[:, None, None] * \
                (t[None, None, :] - pos[None, :, None])
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[r0:r1]).transpose(0, 1),
            torch.from_numpy(k).transpose(0, 1).repeat_interleave(g, 0),
            torch.from_numpy(v).transpose(0, 1).repeat_interleave(g, 0),
            attn_mask=torch.from_numpy(bias), scale=float(W.scale))
        out[r0:r1] = o.transpose(0, 1).numpy()
    return out


def _w(seed=41):
    return wl.build_workload("opt", seed, [1, 7, 1, 30], [50, 7, 16, 90], 4, 2, 16)


def test_window_wider_than_context_is_plain(oracle):
    W = _w()
    kc, vc = oracle_pools(oracle, W)
    assert np.array_equal(oracle_attention(oracle, W, kc, vc),
                          oracle_attention(oracle, W, kc, vc, window=1000))


def test_window_of_one_returns_the_own_value(oracle):
    W = wl.build_workload("w1", 42, [1, 1], [30, 5], 4, 2, 16)
    kc, vc = oracle_pools(oracle, W)
    out = oracle_attention(oracle, W, kc, vc, window=1)
    for r in range(2):
        v = npo.to_f64(W.new_v[r], W.src_dtype)
        for hq in range(4):
            assert np.array_equal(out[r, hq], v[hq // 2])


@pytest.mark.parametrize("window", [1, 5, 16, 17, 33])
def test_window_matches_masked_sdpa(oracle, window):
    W = _w(43)
    kc, vc = oracle_pools(oracle, W)
    np.testing.assert_allclose(oracle_attention(oracle, W, kc, vc, window=window),
                               _reference(W, kc, vc, window=window), rtol=0, atol=1e-12)


def test_zero_alibi_slopes_are_plain(oracle):
    W = _w(44)
    kc, vc = oracle_pools(oracle, W)
    assert np.array_equal(oracle_attention(oracle, W, kc, vc),
                          oracle_attention(oracle, W, kc, vc, alibi_slopes=np.zeros(4, np.float32)))


def test_alibi_matches_biased_sdpa(oracle):
    W = _w(45)
    kc, vc = oracle_pools(oracle, W)
    slopes = np.array([2 ** -1, 2 ** -2, 2 ** -3, 2 ** -4], np.float32)   # ALiBi geometric slopes
    np.testing.assert_allclose(oracle_attention(oracle, W, kc, vc, alibi_slopes=slopes),
                               _reference(W, kc, vc, slopes=slopes), rtol=0, atol=1e-12)
    np.testing.assert_allclose(
        oracle_attention(oracle, W, kc, vc, alibi_slopes=slopes, window=9),
        _reference(W, kc, vc, window=9, slopes=slopes), rtol=0, atol=1e-12)


def test_alibi_and_window_brute_force_tiny(oracle):
    """Two keys, D = 1: closed form with the ALiBi bias written out."""
    bs = 16
    kc = np.zeros((1, 1, bs, 1), np.uint16)
    vc = np.zeros((1, 1, bs, 1), np.uint16)
    kc[0, 0, :3, 0] = [0x3F80, 0x0000, 0x3F80]        # keys 1, 0, 1
    vc[0, 0, :3, 0] = [0x4040, 0x3F80, 0x0000]        # values 3, 1, 0
    q = np.array([[[0x3F80]]], np.uint16)
    s = 0.5
    slope = np.float32(0.25)
    out = oracle.paged_decode(q, wl.BF16, np.array([3], np.int32), kc, vc, wl.BF16,
                              np.array([[0]], np.int32), s, alibi_slopes=np.array([slope]))
    logits = [s * 1 + float(slope) * (0 - 2), s * 0 + float(slope) * (1 - 2), s * 1]
    w = [math.exp(x) for x in logits]
    assert abs(out[0, 0, 0] - (3 * w[0] + 1 * w[1]) / sum(w)) < 1e-15
    out2 = oracle.paged_decode(q, wl.BF16, np.array([3], np.int32), kc, vc, wl.BF16,
                               np.array([[0]], np.int32), s, window=2,
                               alibi_slopes=np.array([slope]))
    w2 = w[1:]
    assert abs(out2[0, 0, 0] - (1 * w2[0]) / sum(w2)) < 1e-15
