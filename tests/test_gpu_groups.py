"""GPU-vs-oracle parity for the GQA group sizes and head dims beyond the
reference workloads' ("PagedAttention 与 Continuous Batching", §10.8: the
paged kernels cover MHA, MQA and GQA): groups of more than 8 query heads per
KV head (MQA 16/1, 32/1, 128/1; GQA 64/4 and a non-power-of-two 24/2) in
decode and in the packed varlen step, the tensor-core chunk path at head_dim
64 and 256, and a step with more chunk work units than the GPU has SMs (each
persistent chunk CTA then runs several units), and E4M3 pools on the chunk
path (K and V widened to f16 in shared memory).
"""
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
LENS = [1, 15, 16, 17, 63, 64, 65, 511, 513, 1000]


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


@pytest.mark.parametrize("hq,hkv,D", [(16, 1, 128), (32, 1, 128), (64, 4, 128), (24, 2, 128),
                                      (128, 1, 64), (32, 2, 256)])
def test_decode_large_groups(oracle, hq, hkv, D):
    W = wl.build_workload("dgrp", 600 + hq + D, np.ones(len(LENS), np.int64), LENS, hq, hkv, D)
    for ps in (0, 64):
        _run(oracle, W, F32, partition_size=ps)


def test_decode_large_group_fp8_and_bf16_out(oracle):
    W = wl.build_workload("dgrp8", 611, np.ones(5, np.int64), [3, 100, 513, 1024, 2000], 32, 2,
                          128, kv_dtype=wl.FP8_E4M3, out_dtype=wl.BF16)
    _run(oracle, W, F32)
    _run(oracle, W, wl.BF16)


@pytest.mark.parametrize("hq,hkv", [(16, 1), (32, 1), (64, 4), (128, 1)])
def test_varlen_large_groups(oracle, hq, hkv):
    """Query tiles of 128/G positions (8, 4, 1 for G = 16, 32, 128), chunk
    starts off the block and key-tile grid, a decode row beside them."""
    q_lens = [1, 37, 130, 3, 64]
    kv_lens = [700, 37 + 50, 130 + 333, 3 + 16, 64]
    W = wl.build_workload("vgrp", 620 + hq, q_lens, kv_lens, hq, hkv, 128)
    _run(oracle, W, F32)


@pytest.mark.parametrize("D", [64, 256])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (32, 8)])
def test_varlen_head_dims_on_the_chunk_path(oracle, D, hq, hkv):
    q_lens = [300, 1, 130, 257, 2]
    kv_lens = [300 + 77, 1000, 130 + 400, 257 + 129, 2 + 61]
    W = wl.build_workload("vdim", 640 + D + hq, q_lens, kv_lens, hq, hkv, D)
    _run(oracle, W, F32)
    _run(oracle, W, wl.BF16)


@pytest.mark.parametrize("D", [64, 256])
def test_varlen_head_dims_window_alibi(oracle, D):
    W = wl.build_workload("vdimw", 660 + D, [200, 1, 90], [200 + 300, 500, 90], 8, 2, D)
    _run(oracle, W, F32, window=100, alibi=True)


def test_varlen_more_units_than_sms(oracle):
    """60 requests with chunks of 40..140 rows over up to 1.5K cached keys, GQA
    32/8: about 80 (request, query-tile pair) items x 8 KV heads = 640 units
    for ~148 persistent CTAs, in heaviest-first order."""
    rng = np.random.default_rng(680)
    q_lens = rng.integers(40, 141, size=60)
    q_lens[::7] = 1                                   # some decode rows among them
    kv_lens = q_lens + rng.integers(0, 1500, size=60)
    W = wl.build_workload("vmany", 680, q_lens, kv_lens, 32, 8, 128)
    _run(oracle, W, F32)
    _run(oracle, W, F32, window=256)


def test_full_size_mqa_decode_sampled(oracle):
    """A full-size Llama-3-8B-shaped batch (256 sequences, lognormal lengths
    with median 1000 in [32, 8192]) with all 32 query heads on one KV head."""
    rng = np.random.default_rng(1003 + 7919)
    lens = np.clip(np.rint(rng.lognormal(math.log(1000.0), 1.0, size=256)), 32, 8192)
    W = wl.build_workload("mqa_full", 1013, np.ones(256, np.int64), lens.astype(np.int64), 32, 1,
                          128, partition_size=512)
    d = DeviceStep(W)
    d.fill_cache()
    d.step()
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    got = d.out_f64()
    assert np.isfinite(got).all()
    L = W.seqlens_k
    rows = sorted({int(np.argmax(L)), int(np.argmin(L)), *rng.choice(256, 6, replace=False)})
    kc, vc = sampled_oracle_pools(oracle, W, rows)
    pr = np.repeat(rows, W.num_q_heads)
    ph = np.tile(np.arange(W.num_q_heads), len(rows))
    want = oracle_attention(oracle, W, kc, vc, pairs=(pr, ph), num_threads=8)
    assert_close(got[pr, ph], want, W, W.out_dtype, W.name)


@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 4), (32, 8)])
@pytest.mark.parametrize("q_dtype", [wl.BF16, wl.F16])
def test_varlen_fp8_pool_on_the_chunk_path(oracle, hq, hkv, q_dtype):
    """E4M3 pools at head_dim 128 run their chunks on the tensor-core kernel
    (K and V widened to f16 in shared memory): chunks of several query tiles
    over cached context off the block and key-tile grid, decode rows beside."""
    q_lens = [300, 1, 130, 257, 2]
    kv_lens = [300 + 77, 1000, 130 + 400, 257 + 129, 2 + 61]
    W = wl.build_workload("v8c", 700 + hq + q_dtype, q_lens, kv_lens, hq, hkv, 128, dtype=q_dtype,
                          kv_dtype=wl.FP8_E4M3, out_dtype=wl.BF16)
    _run(oracle, W, F32)
    _run(oracle, W, wl.BF16)


def test_varlen_fp8_pool_chunks_window_alibi_and_block_sizes(oracle):
    for bs in (8, 16, 32):
        W = wl.build_workload("v8w", 720 + bs, [200, 1, 90], [200 + 300, 500, 90], 8, 2, 128,
                              kv_dtype=wl.FP8_E4M3, block_size=bs)
        _run(oracle, W, F32, window=100, alibi=True)
        _run(oracle, W, F32)
