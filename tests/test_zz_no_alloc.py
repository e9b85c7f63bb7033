"""pa_decode_static: paged decode for callers that cannot allocate device memory.

Such a caller (a plug-in inside a program that owns all device memory, or a
loop that cannot afford cudaMalloc's device-wide synchronisation) cannot hand
pa_decode a workspace, so pa_decode_static keeps its split-K partials in a
fixed device array inside the library.  These checks call it through the C
ABI twice in a row, on two different batches, and compare each result with
pa_decode given an ordinary workspace; the second call must not see anything
the first one left in the shared array.  The file sorts last so that a run
stopping at its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_lens_b200 import pa
from paged_kv_cache_lens_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TD = {wl.F16: torch.float16, wl.BF16: torch.bfloat16, wl.F32: torch.float32}


def _dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(TD[dt])


def _setup(seed, batch, ps):
    """A decode batch whose long rows span several partitions (scratch in use)."""
    W = wl.build_workload("static", seed, np.ones(batch, np.int64),
                          np.random.default_rng(seed).integers(1, 2500, batch), 32, 8, 128,
                          partition_size=ps)
    shape = (W.num_blocks, W.num_kv_heads, W.block_size, W.head_dim)
    kc = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    slots = np.concatenate([W.prefill_slots, W.new_slots])
    pa.pa_reshape_and_cache(_dev(np.concatenate([W.prefill_k, W.new_k]), W.src_dtype),
                            _dev(np.concatenate([W.prefill_v, W.new_v]), W.src_dtype),
                            torch.from_numpy(slots).cuda(), kc, vc)
    return W, kc, vc, _dev(W.q, W.q_dtype), torch.from_numpy(W.block_tables).cuda(), \
        torch.from_numpy(W.seqlens_k).cuda()


def _call_static(lib, out, q, kc, vc, bt, sk, W, ps):
    desc = pa.cache_desc(kc)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.pa_decode_static(
        ctypes.c_void_p(out.data_ptr()), pa.dtype_code(out.dtype), ctypes.c_void_p(q.data_ptr()),
        pa.dtype_code(q.dtype), W.num_seqs, W.num_q_heads, ctypes.c_void_p(kc.data_ptr()),
        ctypes.c_void_p(vc.data_ptr()), ctypes.byref(desc), ctypes.c_void_p(bt.data_ptr()),
        bt.shape[1], ctypes.c_void_p(sk.data_ptr()), W.max_context_len, W.scale, ps, stream)


@pytest.fixture(scope="module")
def lib():
    lib = pa.load_library()
    P, i32, E, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int, ctypes.c_float
    lib.pa_decode_static.argtypes = [P, E, P, E, i32, i32, P, P, ctypes.POINTER(pa.pa_cache_desc),
                                     P, i32, P, i32, F, i32, P]
    lib.pa_decode_static.restype = E
    return lib


def test_static_scratch_matches_pa_decode_on_two_calls(lib):
    torch.cuda.set_device(0)
    for seed, batch, ps in ((71, 24, 256), (72, 40, 128)):
        W, kc, vc, q, bt, sk = _setup(seed, batch, ps)
        need = pa.pa_decode_workspace_size(W.num_seqs, W.num_q_heads, W.head_dim,
                                           W.max_context_len, ps)
        assert 0 < need <= 32 * 1024 * 1024          # the split-K scratch is really used
        ref = torch.empty((W.num_seqs, W.num_q_heads, W.head_dim), dtype=torch.float32,
                          device="cuda")
        pa.pa_decode(ref, q, kc, vc, bt, sk, W.max_context_len, W.scale, partition_size=ps)
        out = torch.full_like(ref, float("nan"))
        assert _call_static(lib, out, q, kc, vc, bt, sk, W, ps) == 0
        torch.cuda.synchronize()
        assert pa.pa_device_error() == 0
        torch.testing.assert_close(out, ref, rtol=0, atol=2e-3)


def test_static_scratch_call_takes_no_device_memory(lib):
    """After the first call (which loads the library's device code, array
    included), a call leaves the device's free memory exactly as it found it:
    it allocates nothing."""
    torch.cuda.set_device(0)
    W, kc, vc, q, bt, sk = _setup(74, 32, 256)
    out = torch.empty((W.num_seqs, W.num_q_heads, W.head_dim), dtype=torch.float32,
                      device="cuda")
    assert _call_static(lib, out, q, kc, vc, bt, sk, W, 256) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _call_static(lib, out, q, kc, vc, bt, sk, W, 256) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert pa.pa_device_error() == 0


def test_static_scratch_rejects_sizes_beyond_its_capacity(lib):
    torch.cuda.set_device(0)
    W, kc, vc, q, bt, sk = _setup(73, 4, 128)
    big_batch = 4096                       # partials for 4096 x 32 heads x 20 parts >> 32 MiB
    out = torch.empty((W.num_seqs, W.num_q_heads, W.head_dim), dtype=torch.float32,
                      device="cuda")
    desc = pa.cache_desc(kc)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.pa_decode_static(
        ctypes.c_void_p(out.data_ptr()), pa.PA_F32, ctypes.c_void_p(q.data_ptr()), pa.PA_BF16,
        big_batch, W.num_q_heads, ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
        ctypes.byref(desc), ctypes.c_void_p(bt.data_ptr()), 160, ctypes.c_void_p(sk.data_ptr()),
        2560, W.scale, 128, stream)
    assert st == 3                          # PA_ERR_WORKSPACE, nothing launched
