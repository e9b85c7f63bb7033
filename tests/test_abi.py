"""The C-ABI library loads on a CPU-only host, exports every entry point its
header declares, and answers the host-only calls (status strings, workspace
sizing, argument validation) without touching a GPU."""
import ctypes
import re

import pytest

from paged_kv_cache_lens_b200 import build as pa_build
from paged_kv_cache_lens_b200 import pa


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return pa.load_library()


def test_header_declares_the_boundary():
    names = pa.declared_functions()
    for n in ["pa_reshape_and_cache", "pa_decode", "pa_varlen", "pa_decode_workspace_size",
              "pa_varlen_workspace_size", "pa_status_string", "pa_device_error"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in pa.declared_functions():
        assert hasattr(lib, name), name


def test_header_is_plain_c():
    text = open(pa.HEADER).read()
    assert 'extern "C"' in text
    for bad in ("torch", "at::", "Tensor", "cuda_runtime", "cudaStream_t"):
        assert bad not in re.sub(r"/\*.*?\*/", "", text, flags=re.S), bad


def test_status_strings(lib):
    for code, name in pa.STATUS_NAMES.items():
        assert pa.pa_status_string(code).startswith(name)
    assert pa.pa_status_string(99) == "PA_ERR_UNKNOWN"


def test_varlen_workspace_ex_sizes_partials_for_the_rows_that_use_them(lib):
    """With the chunk path (a power-of-two group; a 16-bit pool at head_dim
    64/128/256 or an E4M3 pool at 128) only the q_len-1 requests take split-K
    partials, one row each: the exact-type size is the worst-case size
    recomputed with num_seqs rows.  A step of decode rows only, or a q dtype
    other than the pool's 16-bit type, sends every row to the decode kernel:
    then the sizes agree."""
    S, T, H, D, L = 204, 2248, 32, 128, 4097
    worst = pa.pa_varlen_workspace_size(S, T, H, D, L)
    chunk = pa.pa_varlen_workspace_size_ex(S, T, H, 8, D, 512, L, pa.PA_BF16, pa.PA_BF16)
    fp8 = pa.pa_varlen_workspace_size_ex(S, T, H, 8, D, 512, L, pa.PA_BF16, pa.PA_FP8_E4M3)
    mixed_types = pa.pa_varlen_workspace_size_ex(S, T, H, 8, D, 512, L, pa.PA_F16, pa.PA_BF16)
    decode_only = pa.pa_varlen_workspace_size_ex(S, T, H, 8, D, 1, L, pa.PA_BF16, pa.PA_BF16)
    assert mixed_types == worst == decode_only
    assert fp8 == chunk
    assert chunk < 40e6 < worst
    # partials of 204 rows x 32 heads x 9 parts (512 tokens) for m, l and o
    al = lambda x: -(-x // 256) * 256  # noqa: E731
    n = S * H * 9
    head = 2 * al(4 * T) + al(8 * T) + 256
    assert chunk == head + 2 * al(4 * n) + al(4 * n * D)
    assert pa.pa_varlen_workspace_size_ex(S, T, H, 3, D, 512, L, pa.PA_BF16, pa.PA_BF16) == 0


def test_decode_workspace_size_closed_form(lib):
    # one partition (no split) needs no workspace
    assert pa.pa_decode_workspace_size(64, 40, 128, 512, 512) == 0
    # B*Hq*P floats for m and for l, B*Hq*P*D for o, each 256-aligned
    B, H, D, L, P = 64, 40, 128, 2048, 512
    parts = -(-L // P)
    n = B * H * parts

    def al(x):
        return -(-x // 256) * 256
    assert pa.pa_decode_workspace_size(B, H, D, L, P) == 2 * al(4 * n) + al(4 * n * D)
    assert pa.pa_decode_workspace_size(B, H, D, L, 100) == 0     # invalid partition size
    assert pa.pa_decode_workspace_size(0, H, D, L, P) == 0


def test_varlen_workspace_size_includes_row_maps(lib):
    got = pa.pa_varlen_workspace_size(204, 2248, 32, 128, 3584)
    assert got >= 2 * 2248 * 4


def _desc(**kw):
    d = dict(num_blocks=64, block_size=16, num_kv_heads=2, head_dim=64, kv_dtype=pa.PA_F16,
             k_scale=None, v_scale=None)
    d.update(kw)
    return pa.pa_cache_desc(**d)


def test_host_validation_rejects_before_any_launch(lib):
    P = ctypes.c_void_p
    fake = P(0x10000)       # never dereferenced: every call below fails validation first
    desc = _desc()
    # null output
    assert lib.pa_decode(None, 0, fake, 0, 4, 2, fake, fake, ctypes.byref(desc), fake, 8, fake,
                         100, 0.125, 0, None, 0, None) == 1
    # block size other than 8, 16 or 32
    bad = _desc(block_size=64)
    assert lib.pa_decode(fake, 0, fake, 0, 4, 2, fake, fake, ctypes.byref(bad), fake, 8, fake,
                         100, 0.125, 0, None, 0, None) == 2
    # table too narrow for max_context_len
    assert lib.pa_decode(fake, 0, fake, 0, 4, 2, fake, fake, ctypes.byref(desc), fake, 6, fake,
                         100, 0.125, 0, None, 0, None) == 1
    # q heads not a multiple of kv heads
    assert lib.pa_decode(fake, 0, fake, 0, 4, 3, fake, fake, ctypes.byref(desc), fake, 8, fake,
                         100, 0.125, 0, None, 0, None) == 1
    # a group of more than 128 query heads per KV head is not built
    assert lib.pa_decode(fake, 0, fake, 0, 4, 512, fake, fake, ctypes.byref(desc), fake, 8, fake,
                         100, 0.125, 0, None, 0, None) == 2
    # q dtype differs from a 16-bit pool
    assert lib.pa_decode(fake, 0, fake, 1, 4, 2, fake, fake, ctypes.byref(desc), fake, 8, fake,
                         100, 0.125, 0, None, 0, None) == 2
    # bad partition size
    assert lib.pa_decode(fake, 0, fake, 0, 4, 2, fake, fake, ctypes.byref(desc), fake, 8, fake,
                         100, 0.125, 96, None, 0, None) == 1
    # workspace needed (4 parts of 64) but missing
    assert lib.pa_decode(fake, 0, fake, 0, 4, 2, fake, fake, ctypes.byref(desc), fake, 8, fake,
                         100, 0.125, 64, None, 0, None) == 3
    # FP8 pool without scales
    f8 = _desc(kv_dtype=pa.PA_FP8_E4M3, head_dim=128)
    assert lib.pa_decode(fake, 1, fake, 1, 4, 2, fake, fake, ctypes.byref(f8), fake, 8, fake,
                         100, 0.125, 0, None, 0, None) == 1
    # misaligned pool
    assert lib.pa_decode(fake, 0, fake, 0, 4, 2, P(0x10002), fake, ctypes.byref(desc), fake, 8,
                         fake, 100, 0.125, 0, None, 0, None) == 1
    # reshape: stride smaller than a row, unsupported dtype pair
    assert lib.pa_reshape_and_cache(fake, fake, 0, 4, 8, fake, fake, fake, ctypes.byref(desc),
                                    None) == 1
    assert lib.pa_reshape_and_cache(fake, fake, 1, 4, 128, fake, fake, fake, ctypes.byref(desc),
                                    None) == 2
    # zero work is a no-op success
    assert lib.pa_reshape_and_cache(fake, fake, 0, 0, 128, fake, fake, fake, ctypes.byref(desc),
                                    None) == 0
    assert lib.pa_decode(fake, 0, fake, 0, 0, 2, fake, fake, ctypes.byref(desc), fake, 8, fake,
                         100, 0.125, 0, None, 0, None) == 0
    # varlen: workspace missing, q longer than context
    assert lib.pa_varlen(fake, 0, fake, 0, 10, 2, 2, fake, fake, 5, 100, fake, fake,
                         ctypes.byref(desc), fake, 8, 0.125, None, 0, None) == 3
    assert lib.pa_varlen(fake, 0, fake, 0, 10, 2, 2, fake, fake, 200, 100, fake, fake,
                         ctypes.byref(desc), fake, 8, 0.125, None, 0, None) == 1


def test_block_ops_and_probe_validation(lib):
    """Host-side checks of the block operations, the options struct and the
    read probe: each case fails (or succeeds with no work) before any launch."""
    import numpy as np
    P = ctypes.c_void_p
    fake = P(0x10000)
    desc = _desc()
    # copy_blocks: negative count, no pairs (a no-op), missing mapping, f32 pool,
    # blocks that are not a whole number of 16-byte units
    assert lib.pa_copy_blocks(fake, fake, ctypes.byref(desc), fake, -1, None) == 1
    assert lib.pa_copy_blocks(fake, fake, ctypes.byref(desc), fake, 0, None) == 0
    assert lib.pa_copy_blocks(fake, fake, ctypes.byref(desc), None, 3, None) == 1
    assert lib.pa_copy_blocks(fake, fake, ctypes.byref(_desc(kv_dtype=pa.PA_F32)), fake, 3,
                              None) == 2
    odd = _desc(kv_dtype=pa.PA_FP8_E4M3, head_dim=1, block_size=8, num_kv_heads=1)
    assert lib.pa_copy_blocks(fake, fake, ctypes.byref(odd), fake, 3, None) == 1
    # swap_blocks: a pair outside either pool is caught on the host
    m = np.array([[0, 1], [5, 2]], np.int64)
    mp = m.ctypes.data_as(P)
    assert lib.pa_swap_blocks(fake, fake, fake, fake, ctypes.byref(desc), 4, 8, mp, 2, None) == 1
    assert lib.pa_swap_blocks(fake, fake, fake, fake, ctypes.byref(desc), 8, 2, mp, 2, None) == 1
    assert lib.pa_swap_blocks(fake, fake, fake, fake, ctypes.byref(desc), 8, 8, mp, 0, None) == 0
    assert lib.pa_swap_blocks(fake, fake, fake, fake, ctypes.byref(desc), 8, 8, mp, -1, None) == 1
    # options: ALiBi slopes must be a 4-byte aligned float array
    opts = pa.pa_attn_options(window=0, alibi_slopes=0x10002)
    assert lib.pa_decode_ex(fake, 0, fake, 0, 4, 2, fake, fake, ctypes.byref(desc), fake, 8, fake,
                            100, 0.125, 0, ctypes.byref(opts), None, 0, None) == 1
    # read probe: sizes in 16-byte units, aligned buffer and sink
    assert lib.pa_hbm_read_probe(fake, 24, fake, None) == 1
    assert lib.pa_hbm_read_probe(fake, -16, fake, None) == 1
    assert lib.pa_hbm_read_probe(fake, 32, None, None) == 1
    assert lib.pa_hbm_read_probe(P(0x10008), 32, fake, None) == 1


def test_static_decode_and_varlen_options_validation(lib):
    """Refusals that come before any CUDA call: pa_decode_static without a
    pool description or with partials past its fixed scratch, and pa_varlen_ex
    with ALiBi slopes that are not a 4-byte aligned float array."""
    P, i32, E, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int, ctypes.c_float
    lib.pa_decode_static.argtypes = [P, E, P, E, i32, i32, P, P, ctypes.POINTER(pa.pa_cache_desc),
                                     P, i32, P, i32, F, i32, P]
    lib.pa_decode_static.restype = E
    fake = P(0x10000)
    desc = _desc()
    assert lib.pa_decode_static(fake, 0, fake, 0, 4, 2, fake, fake, None, fake, 8, fake, 100,
                                0.125, 0, None) == 1
    # 4096 rows x 32 heads x 20 partitions of partials: far past 32 MiB
    big = _desc(num_kv_heads=8, head_dim=128, num_blocks=4096)
    assert lib.pa_decode_static(fake, 0, fake, 0, 4096, 32, fake, fake, ctypes.byref(big), fake,
                                160, fake, 2560, 0.125, 128, None) == 3
    opts = pa.pa_attn_options(window=0, alibi_slopes=0x10002)
    assert lib.pa_varlen_ex(fake, 0, fake, 0, 10, 2, 2, fake, fake, 5, 100, fake, fake,
                            ctypes.byref(desc), fake, 8, 0.125, ctypes.byref(opts), fake, 1 << 40,
                            None) == 1
