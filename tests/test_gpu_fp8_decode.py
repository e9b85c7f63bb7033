"""GPU-vs-oracle parity of decode over E4M3 pools at head_dim 128 with many
(row, KV head, partition) work items per launch: single-partition batches of
hundreds of rows, split-K partitions of 64..1024 keys (partial tiles,
partitions that end inside a tile), sliding windows that leave whole
partitions invisible, ALiBi, 8/16/32-token blocks, queries with a large
dynamic range, the full shared-prefix workload sampled, and a workspace
reused across calls ("PagedAttention 与 Continuous Batching", §3.6
PagedAttention Kernel; split-K partitions and their log-sum-exp merge)."""
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_lens_b200 import pa
from paged_kv_cache_lens_b200 import workloads as wl
from tests._gpu import DeviceStep, assert_close, sampled_oracle_pools
from tests._helpers import oracle_attention, oracle_pools

pytestmark = pytest.mark.gpu

F32 = wl.F32


def _run(oracle, W, out_dtype=F32, partition_size=None, window=0, alibi=False):
    d = DeviceStep(W, out_dtype=out_dtype)
    d.fill_cache()
    slopes = None
    if alibi:
        slopes = np.array([2.0 ** (-8.0 * (i + 1) / W.num_q_heads) for i in range(W.num_q_heads)],
                          np.float32)
        d.alibi = torch.from_numpy(slopes).cuda()
    d.window = window
    d.step(partition_size=partition_size)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    kc, vc = oracle_pools(oracle, W)
    want = oracle_attention(oracle, W, kc, vc, window=window, alibi_slopes=slopes)
    return assert_close(d.out_f64(), want, W, out_dtype, W.name)


@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (24, 8), (64, 8)])
def test_single_partition_many_units_per_cta(oracle, hq, hkv):
    """Contexts of at most 512 keys, 300 rows: one partition per row."""
    rng = np.random.default_rng(900 + hq)
    lens = rng.integers(1, 513, size=300)
    lens[::97] = 512
    W = wl.build_workload("tc1", 900 + hq, np.ones(300, np.int64), lens, hq, hkv, 128,
                          kv_dtype=wl.FP8_E4M3, out_dtype=wl.BF16)
    _run(oracle, W, F32)


@pytest.mark.parametrize("ps", [0, 64, 192, 1024])
def test_split_partitions_many_units_per_cta(oracle, ps):
    """Long contexts in partitions of 64..1024 keys (partial last tiles)."""
    rng = np.random.default_rng(910 + ps)
    lens = rng.integers(1, 3000, size=64)
    lens[:3] = [1, 127, 2999]
    W = wl.build_workload("tc2", 910 + ps, np.ones(64, np.int64), lens, 32, 8, 128,
                          kv_dtype=wl.FP8_E4M3, dtype=wl.F16)
    _run(oracle, W, F32 if ps in (0, 192) else wl.BF16, partition_size=ps)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_window_alibi_and_block_sizes(oracle, bs):
    """A sliding window that leaves whole partitions invisible, and ALiBi,
    over 8-, 16- and 32-token blocks."""
    rng = np.random.default_rng(920 + bs)
    lens = rng.integers(1, 2500, size=64)
    W = wl.build_workload("tc3", 920 + bs, np.ones(64, np.int64), lens, 32, 8, 128,
                          kv_dtype=wl.FP8_E4M3, block_size=bs)
    _run(oracle, W, F32, window=700, alibi=True)
    _run(oracle, W, F32, partition_size=256, window=300)


def test_query_rows_with_large_dynamic_range(oracle):
    """q whose elements span 2^-12 .. 2^4 per head, an all-zero head and one
    element near 900."""
    lens = np.random.default_rng(930).integers(100, 2000, size=64)
    for q_dtype in (wl.BF16, wl.F16):
        W = wl.build_workload("tc4", 930 + q_dtype, np.ones(64, np.int64), lens, 32, 8, 128,
                              dtype=q_dtype, kv_dtype=wl.FP8_E4M3)
        rng = np.random.default_rng(931 + q_dtype)
        q = rng.standard_normal((W.total_q, 32, 128)).astype(np.float32)
        q *= np.exp2(rng.uniform(-12, 4, size=q.shape)).astype(np.float32)
        q[:, 1, :] = 0.0
        q[:, 6, 7] = 900.0
        W.q = wl.f32_to_bf16_bits(q) if q_dtype == wl.BF16 else q.astype(np.float16).view(np.uint16)
        _run(oracle, W, F32)


def test_full_size_shared_prefix_fp8_sampled(oracle):
    """The full shared-prefix workload (128 sequences, 2048 shared keys +
    U[0, 6144] private ones, 32/8 heads) in the launch configuration the
    benchmark times; sampled rows against the oracle, all rows finite."""
    W = wl.config(5)
    d = DeviceStep(W)
    d.fill_cache()
    d.step()
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    got = d.out_f64()
    assert np.isfinite(got).all()
    L = W.seqlens_k
    rng = np.random.default_rng(5)
    rows = sorted({int(np.argmax(L)), int(np.argmin(L)), *rng.choice(W.num_seqs, 6, replace=False)})
    kc, vc = sampled_oracle_pools(oracle, W, rows)
    pr = np.repeat(rows, W.num_q_heads)
    ph = np.tile(np.arange(W.num_q_heads), len(rows))
    want = oracle_attention(oracle, W, kc, vc, pairs=(pr, ph), num_threads=8)
    assert_close(got[pr, ph], want, W, W.out_dtype, W.name)


def test_repeated_steps_reuse_the_workspace(oracle):
    """Two calls on one workspace give identical results (the second sees the
    first's partials)."""
    lens = np.random.default_rng(940).integers(1, 3000, size=48)
    W = wl.build_workload("tc5", 940, np.ones(48, np.int64), lens, 32, 8, 128,
                          kv_dtype=wl.FP8_E4M3)
    d = DeviceStep(W)
    d.fill_cache()
    d.step()
    first = d.out_f64().copy()
    d.out.fill_(float("nan"))
    d.step()
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    assert np.array_equal(first, d.out_f64())
    kc, vc = oracle_pools(oracle, W)
    assert_close(first, oracle_attention(oracle, W, kc, vc), W, F32, W.name)
    assert math.isfinite(float(np.abs(first).max()))
