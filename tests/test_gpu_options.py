"""GPU parity of the sliding-window and ALiBi variants (pa_decode_ex /
pa_varlen_ex) against the oracle: decode (bf16, FP8, several partitions),
and packed varlen steps whose chunks run on the tensor-core prefill kernel."""
import numpy as np
import pytest
import torch

from paged_kv_cache_lens_b200 import pa
from paged_kv_cache_lens_b200 import workloads as wl
from tests._gpu import DeviceStep, assert_close
from tests._helpers import oracle_attention, oracle_pools

pytestmark = pytest.mark.gpu


def _slopes(hq):
    # the ALiBi geometric sequence 2^(-8 i / H)
    return np.array([2.0 ** (-8.0 * (i + 1) / hq) for i in range(hq)], np.float32)


def _run(oracle, W, window, alibi, partition_size=None):
    d = DeviceStep(W, out_dtype=wl.F32)
    d.window = window
    d.alibi = torch.from_numpy(alibi).cuda() if alibi is not None else None
    d.fill_cache()
    d.step(partition_size=partition_size)
    torch.cuda.synchronize()
    assert pa.pa_device_error() == 0
    kc, vc = oracle_pools(oracle, W)
    want = oracle_attention(oracle, W, kc, vc, window=window, alibi_slopes=alibi)
    return assert_close(d.out_f64(), want, W, wl.F32, W.name)


@pytest.mark.parametrize("window", [1, 17, 100, 600])
@pytest.mark.parametrize("use_alibi", [False, True])
@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 4)])
def test_decode_window_alibi(oracle, window, use_alibi, hq, hkv):
    lens = [1, 16, 17, 100, 513, 1500]
    W = wl.build_workload("wd", 600 + window + hq, np.ones(len(lens), np.int64), lens, hq, hkv,
                          128)
    for ps in (0, 64):
        _run(oracle, W, window, _slopes(hq) if use_alibi else None, partition_size=ps)


def test_decode_alibi_only(oracle):
    W = wl.build_workload("ad", 610, np.ones(4, np.int64), [3, 200, 900, 2100], 32, 8, 128)
    _run(oracle, W, 0, _slopes(32))


def test_decode_fp8_window(oracle):
    W = wl.build_workload("wf8", 611, np.ones(4, np.int64), [40, 300, 900, 1300], 8, 2, 128,
                          kv_dtype=wl.FP8_E4M3)
    _run(oracle, W, 250, _slopes(8))


@pytest.mark.parametrize("window", [0, 1, 40, 300])
@pytest.mark.parametrize("use_alibi", [False, True])
def test_varlen_window_alibi(oracle, window, use_alibi):
    q_lens = [1, 300, 1, 130, 40]
    kv_lens = [700, 300 + 77, 33, 130 + 500, 40]
    for hq, hkv in [(32, 8), (8, 8)]:
        W = wl.build_workload("wv", 620 + window + hq, q_lens, kv_lens, hq, hkv, 128)
        if window == 0 and not use_alibi:
            continue
        _run(oracle, W, window, _slopes(hq) if use_alibi else None)
