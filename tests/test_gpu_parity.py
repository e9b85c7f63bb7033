"""GPU-vs-oracle parity of the hot path, called through the C ABI.

Cache writes and indexing must match the oracle bit for bit; attention must
be within max-abs 2e-3 (fp16/bf16 pools) or 5e-2 (FP8 pools) of the fp64
oracle with fp32 output, plus half an output ulp when the output is 16-bit.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_lens_b200 import pa
from paged_kv_cache_lens_b200 import workloads as wl
from tests._gpu import DeviceStep, assert_close, sampled_oracle_pools
from tests._helpers import oracle_attention, oracle_pools

pytestmark = pytest.mark.gpu

F32 = wl.F32


def _pool_bits(t):
    return t.view(torch.uint8).cpu().numpy() if t.dtype == torch.uint8 else \
        t.view(torch.int16).cpu().numpy().view(np.uint16)


def _run_small(oracle, W, out_dtype=F32, partition_size=None):
    d = DeviceStep(W, out_dtype=out_dtype)
    d.fill_cache()
    d.step(partition_size=partition_size)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    kc, vc = oracle_pools(oracle, W)
    assert np.array_equal(_pool_bits(d.k_cache), kc), "K pool differs from the oracle's"
    assert np.array_equal(_pool_bits(d.v_cache), vc), "V pool differs from the oracle's"
    want = oracle_attention(oracle, W, kc, vc)
    got = d.out_f64()
    return assert_close(got, want, W, out_dtype, W.name), d


# ---------------------------------------------------------------- cache write

@pytest.mark.parametrize("kv", [wl.BF16, wl.F16, wl.FP8_E4M3])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_reshape_and_cache_bit_exact(oracle, kv, bs):
    W = wl.build_workload("rc", 101, [1, 1, 1, 7], [1, 30, 64, 100], 8, 4, 128,
                          dtype=wl.F16 if kv == wl.F16 else wl.BF16, kv_dtype=kv, block_size=bs)
    W.new_slots[2] = -1                          # a padding token is skipped
    d = DeviceStep(W)
    d.fill_cache()
    d.write_new()
    torch.cuda.synchronize()
    kc, vc = oracle_pools(oracle, W)
    assert np.array_equal(_pool_bits(d.k_cache), kc)
    assert np.array_equal(_pool_bits(d.v_cache), vc)


def test_reshape_and_cache_from_fused_qkv_rows(oracle):
    rng = np.random.default_rng(7)
    T, hq, hkv, D, nb = 37, 8, 2, 64, 16
    qkv = wl.randn_bits(rng, (T, (hq + 2 * hkv) * D), wl.BF16)
    slots = rng.choice(nb * 16, T, replace=False).astype(np.int64)
    dev = torch.from_numpy(qkv.view(np.int16)).cuda().view(torch.bfloat16)
    k = dev[:, hq * D:(hq + hkv) * D].view(T, hkv, D)
    v = dev[:, (hq + hkv) * D:].view(T, hkv, D)
    kc = torch.zeros((nb, hkv, 16, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    pa.pa_reshape_and_cache(k, v, torch.from_numpy(slots).cuda(), kc, vc)
    ok_, ov_ = np.zeros((nb, hkv, 16, D), np.uint16), np.zeros((nb, hkv, 16, D), np.uint16)
    oracle.reshape_and_cache(qkv[:, hq * D:], qkv[:, (hq + hkv) * D:], wl.BF16, slots, ok_, ov_,
                             16, wl.BF16, token_stride=(hq + 2 * hkv) * D)
    assert np.array_equal(_pool_bits(kc), ok_) and np.array_equal(_pool_bits(vc), ov_)


# ---------------------------------------------------------------- decode

def test_config1_tiny_mha_all_outputs(oracle):
    W = wl.config(1)
    for out_dtype in (F32, wl.F16):
        _run_small(oracle, W, out_dtype)


EDGE_LENS = [1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 511, 512, 513, 1000]


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (16, 2), (6, 2)])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_decode_edge_lengths(oracle, hq, hkv, D):
    W = wl.build_workload("edge", 200 + D + hq, np.ones(len(EDGE_LENS), np.int64), EDGE_LENS, hq,
                          hkv, D, dtype=wl.BF16)
    for ps in (0, 64, 512):
        _run_small(oracle, W, F32, partition_size=ps)


@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("hq,hkv,D", [(4, 4, 64), (8, 2, 128), (16, 2, 256)])
def test_decode_block_sizes(oracle, bs, hq, hkv, D):
    """8- and 32-token blocks ("PagedAttention 与 Continuous Batching", §3.7
    block_size 的取舍: 8, 16 or 32), with edge lengths around both sizes."""
    lens = [1, 7, 8, 9, 31, 32, 33, 100, 511, 513]
    W = wl.build_workload("bs", 500 + bs + D, np.ones(len(lens), np.int64), lens, hq, hkv, D,
                          block_size=bs)
    for ps in (0, 64):
        _run_small(oracle, W, F32, partition_size=ps)


@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("D", [64, 128])
def test_decode_fp8_block_sizes(oracle, bs, D):
    W = wl.build_workload("bs8", 510 + bs + D, np.ones(4, np.int64), [5, 40, 700, 1111], 8, 2, D,
                          kv_dtype=wl.FP8_E4M3, block_size=bs)
    _run_small(oracle, W, F32)


@pytest.mark.parametrize("bs", [8, 32])
def test_varlen_block_sizes(oracle, bs):
    q_lens = [1, 130, 1, 257, 33]
    kv_lens = [77, 130 + 45, 999, 257 + 300, 33]
    for hq, hkv in [(32, 8), (4, 4)]:
        W = wl.build_workload("vbs", 520 + bs + hq, q_lens, kv_lens, hq, hkv, 128, block_size=bs)
        _run_small(oracle, W, F32)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("q_dtype", [wl.BF16, wl.F16])
def test_decode_fp8_pool(oracle, D, q_dtype):
    W = wl.build_workload("fp8", 300 + D, np.ones(6, np.int64), [1, 17, 100, 513, 1024, 2000], 8,
                          2, D, dtype=q_dtype, kv_dtype=wl.FP8_E4M3, out_dtype=wl.BF16)
    for out_dtype in (F32, wl.BF16):
        _run_small(oracle, W, out_dtype)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("q_dtype", [wl.BF16, wl.F16])
def test_decode_fp8_query_dynamic_range(oracle, D, q_dtype):
    """E4M3 pool: the query enters QK^T as E4M3 hi + lo parts of q * 2^e, one
    power of two per head.  Heads whose elements span 2^-12 .. 2^4, an
    all-zero head, a head of tiny values and a head with one element near
    the 16-bit formats' 900 still match the oracle."""
    W = wl.build_workload("fp8q", 350 + D, np.ones(4, np.int64), [9, 200, 777, 1500], 8, 2, D,
                          dtype=q_dtype, kv_dtype=wl.FP8_E4M3)
    rng = np.random.default_rng(D + q_dtype)
    q = rng.standard_normal((W.total_q, 8, D)).astype(np.float32)
    q *= np.exp2(rng.uniform(-12, 4, size=q.shape)).astype(np.float32)
    q[:, 1, :] = 0.0
    q[:, 2, :] *= np.float32(2.0 ** -20)
    q[:, 5, 7] = 900.0
    if q_dtype == wl.BF16:
        W.q = wl.f32_to_bf16_bits(q)
    else:
        W.q = q.astype(np.float16).view(np.uint16)
    _run_small(oracle, W, F32)


def test_decode_f16(oracle):
    W = wl.build_workload("f16", 77, np.ones(5, np.int64), [3, 40, 300, 700, 1500], 32, 8, 128,
                          dtype=wl.F16)
    _run_small(oracle, W, F32)
    _run_small(oracle, W, wl.F16)


def test_single_key_returns_value_exactly():
    W = wl.build_workload("one", 5, np.ones(3, np.int64), [1, 1, 1], 8, 2, 128)
    d = DeviceStep(W, out_dtype=wl.BF16)
    d.fill_cache()
    d.step()
    torch.cuda.synchronize()
    got = d.out.view(torch.int16).cpu().numpy().view(np.uint16)     # [3, 8, 128]
    want = np.repeat(W.new_v, 4, axis=1)                              # KV head per group
    assert np.array_equal(got, want)


def test_zero_context_gives_zeros(oracle):
    W = wl.build_workload("z", 6, np.ones(3, np.int64), [5, 40, 9], 4, 2, 64)
    W.seqlens_k[1] = 0
    _, d = _run_small(oracle, W, F32)
    assert torch.all(d.out[1] == 0)


def test_shared_prefix_equals_unshared_copies():
    W = wl.build_workload("sp", 8, np.ones(4, np.int64), [300, 700, 513, 2048], 8, 2, 128,
                          shared_prefix_len=256)
    d = DeviceStep(W, out_dtype=F32)
    d.fill_cache()
    d.step()
    shared = d.out.clone()
    # copy the shared prefix blocks of requests 1..3 into fresh blocks
    nb = W.num_blocks
    extra = 3 * 16
    kc = torch.cat([d.k_cache, torch.zeros((extra,) + d.k_cache.shape[1:], dtype=d.k_cache.dtype,
                                           device="cuda")])
    vc = torch.cat([d.v_cache, torch.zeros_like(kc[:extra])])
    bt = W.block_tables.copy()
    for j, r in enumerate([1, 2, 3]):
        for i in range(16):
            kc[nb + 16 * j + i] = kc[bt[r, i]]
            vc[nb + 16 * j + i] = vc[bt[r, i]]
            bt[r, i] = nb + 16 * j + i
    out2 = torch.empty_like(d.out)
    pa.pa_decode(out2, d.q, kc, vc, torch.from_numpy(bt).cuda(), d.seqlens_k, W.max_context_len,
                 W.scale, workspace=d.workspace)
    torch.cuda.synchronize()
    assert torch.equal(shared, out2)


def test_decode_is_deterministic(oracle):
    W = wl.config(3, batch=16)
    d = DeviceStep(W, out_dtype=F32)
    d.fill_cache()
    d.step()
    a = d.out.clone()
    d.attend()
    torch.cuda.synchronize()
    assert torch.equal(a, d.out)


# ---------------------------------------------------------------- varlen

def test_varlen_small_mixed(oracle):
    q_lens = [1, 5, 17, 1, 33, 3, 64, 1, 100]
    kv_lens = [1, 5, 50, 16, 33, 70, 64, 900, 611]     # chunk starts not multiples of 16
    for hq, hkv, D in [(8, 2, 128), (4, 4, 64), (16, 2, 128), (8, 8, 128), (8, 4, 128)]:
        W = wl.build_workload("vl", 400 + hq, q_lens, kv_lens, hq, hkv, D)
        _run_small(oracle, W, F32)
        _run_small(oracle, W, wl.BF16)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (32, 8), (16, 2)])
def test_varlen_long_chunks(oracle, hq, hkv):
    """Chunks longer than one query tile, over cached context that is not a
    multiple of the block or key-tile size, with a decode row beside them."""
    q_lens = [300, 1, 130, 257]
    kv_lens = [300 + 77, 1000, 130 + 400, 257 + 129]
    W = wl.build_workload("vlong", 420 + hq, q_lens, kv_lens, hq, hkv, 128)
    _run_small(oracle, W, F32)


def test_varlen_fp8(oracle):
    W = wl.build_workload("vl8", 410, [1, 40, 1, 77], [600, 40, 33, 1100], 8, 2, 128,
                          kv_dtype=wl.FP8_E4M3)
    _run_small(oracle, W, F32)


def test_varlen_decode_rows_equal_pa_decode():
    """A varlen batch of q_len-1 requests reproduces pa_decode exactly."""
    W = wl.config(3, batch=12)
    d = DeviceStep(W, out_dtype=F32)
    d.fill_cache()
    d.step()
    dec = d.out.clone()
    out = torch.empty_like(dec)
    pa.pa_varlen(out, d.q, d.cu, d.seqlens_k, 1, W.max_context_len, d.k_cache, d.v_cache,
                 d.block_tables, W.scale)
    torch.cuda.synchronize()
    torch.testing.assert_close(out, dec, rtol=0, atol=2e-5)


# ---------------------------------------------------------------- full sizes

def _sample_rows(W, n, rng):
    L = W.seqlens_k
    picks = {int(np.argmax(L)), int(np.argmin(L))}
    picks.update(int(x) for x in rng.choice(W.num_seqs, min(n, W.num_seqs), replace=False))
    return sorted(picks)


@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_full_size_decode_sampled(oracle, cfg):
    """The reference workload at full size in the benchmark's launch
    configuration; every output finite, sampled (row, head) pairs vs oracle."""
    W = wl.config(cfg)
    d = DeviceStep(W)
    d.fill_cache()
    d.step()
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    got = d.out_f64()
    assert np.isfinite(got).all()
    rng = np.random.default_rng(cfg)
    rows = _sample_rows(W, 6, rng)
    kc, vc = sampled_oracle_pools(oracle, W, rows)
    pr = np.repeat(rows, W.num_q_heads)
    ph = np.tile(np.arange(W.num_q_heads), len(rows))
    want = oracle_attention(oracle, W, kc, vc, pairs=(pr, ph), num_threads=8)
    assert_close(got[pr, ph], want, W, W.out_dtype, W.name)
    _assert_visible_slots_equal(d, W, kc, vc, rows)


def _assert_visible_slots_equal(d, W, kc, vc, rows):
    """Every slot a sampled request's attention reads holds, bit for bit, what
    the oracle's cache write put there (full-size pools, written in pieces by
    pa_reshape_and_cache)."""
    reqs = sorted({int(np.searchsorted(W.cu_seqlens_q, r, side="right") - 1) for r in rows})
    for rq in reqs:
        t = np.arange(int(W.seqlens_k[rq]))
        blk = W.block_tables[rq, t // W.block_size].astype(np.int64)
        off = t % W.block_size
        idx = torch.from_numpy(blk).cuda(), torch.from_numpy(off).cuda()
        for dev_pool, host_pool in ((d.k_cache, kc), (d.v_cache, vc)):
            got = _pool_bits(dev_pool[idx[0], :, idx[1], :])        # [L, Hkv, D]
            assert np.array_equal(got, host_pool[blk, :, off, :]), f"request {rq}"


def test_full_size_mixed_step_sampled(oracle):
    W = wl.config(4)
    d = DeviceStep(W)
    d.fill_cache()
    d.step()
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    got = d.out_f64()
    assert np.isfinite(got).all()
    rng = np.random.default_rng(4)
    dec_rows = sorted(rng.choice(200, 5, replace=False).tolist())
    chunk_rows = []
    for r in range(200, 204):
        base = int(W.cu_seqlens_q[r])
        chunk_rows += [base + i for i in (0, 1, 15, 16, 17, 255, 510, 511)]
    rows = dec_rows + chunk_rows
    kc, vc = sampled_oracle_pools(oracle, W, rows)
    heads = [0, 3, 4, 17, 31]
    pr = np.repeat(rows, len(heads))
    ph = np.tile(heads, len(rows))
    want = oracle_attention(oracle, W, kc, vc, pairs=(pr, ph), num_threads=8)
    assert_close(got[pr, ph], want, W, W.out_dtype, W.name)
    _assert_visible_slots_equal(d, W, kc, vc, rows)


# ---------------------------------------------------------------- errors

def test_out_of_range_block_is_skipped_and_reported():
    W = wl.build_workload("oob", 9, np.ones(2, np.int64), [40, 40], 4, 2, 64)
    d = DeviceStep(W, out_dtype=F32)
    d.fill_cache()
    d.write_new()
    bt = d.block_tables.clone()
    bt[1, 1] = W.num_blocks + 5
    pa.pa_decode(d.out, d.q, d.k_cache, d.v_cache, bt, d.seqlens_k, W.max_context_len, W.scale,
                 workspace=d.workspace)
    assert pa.pa_device_error() == 4
    assert pa.pa_device_error() == 0                       # cleared by the read
    assert torch.isfinite(d.out).all()


def test_out_of_range_slot_is_skipped_and_reported():
    W = wl.build_workload("oobs", 10, [1], [5], 2, 2, 64)
    d = DeviceStep(W)
    bad = torch.tensor([W.num_blocks * 16 + 3], dtype=torch.int64, device="cuda")
    pa.pa_reshape_and_cache(d.new_k, d.new_v, bad, d.k_cache, d.v_cache)
    assert pa.pa_device_error() == 4


def test_row_longer_than_max_context_len_is_cut_and_reported(oracle):
    """A context_lens / seqlens_k entry above the promised max_context_len is
    cut to max_context_len keys and reported as PA_ERR_OUT_OF_RANGE."""
    W = wl.build_workload("cut", 12, np.ones(3, np.int64), [100, 300, 150], 4, 2, 64)
    d = DeviceStep(W, out_dtype=F32)
    d.fill_cache()
    d.write_new()
    torch.cuda.synchronize()
    kc, vc = oracle_pools(oracle, W)
    cut = 200
    pa.pa_decode(d.out, d.q, d.k_cache, d.v_cache, d.block_tables, d.seqlens_k, cut, W.scale,
                 partition_size=64, workspace=None)
    assert pa.pa_device_error() == 4
    want = oracle.paged_attention(W.q, W.q_dtype, W.cu_seqlens_q,
                                  np.minimum(W.seqlens_k, cut).astype(np.int32), kc, vc,
                                  W.kv_dtype, W.block_tables, W.scale)
    assert_close(d.out_f64(), want, W, F32, "cut decode")
    # the packed step: a request with q_len 2 and one with q_len 1, both too long
    V = wl.build_workload("cutv", 13, [2, 1], [180, 300], 8, 2, 128)
    e = DeviceStep(V, out_dtype=F32)
    e.fill_cache()
    e.write_new()
    torch.cuda.synchronize()
    kc, vc = oracle_pools(oracle, V)
    pa.pa_varlen(e.out, e.q, e.cu, e.seqlens_k, V.max_q_len, 160, e.k_cache, e.v_cache,
                 e.block_tables, V.scale)
    assert pa.pa_device_error() == 4
    assert torch.isfinite(e.out).all()


def test_a_wait_that_runs_out_is_reported_and_the_context_survives(oracle):
    """The bounded-wait path: a kernel whose wait can never complete gives up
    after its limit, records PA_ERR_TIMEOUT and returns; the error word reads
    back once, and the next attention call on the same context is correct."""
    pa.pa_selftest_wait_timeout()
    assert pa.pa_device_error() == 6
    assert pa.pa_device_error() == 0
    _run_small(oracle, wl.config(1), F32)


def test_workspace_too_small_is_rejected():
    W = wl.build_workload("ws", 11, np.ones(2, np.int64), [2000, 3000], 8, 2, 128)
    d = DeviceStep(W)
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(d.out, d.q, d.k_cache, d.v_cache, d.block_tables, d.seqlens_k,
                     W.max_context_len, W.scale, partition_size=512, workspace=small)
    assert e.value.status == 3
