"""ctypes front end of the C oracle (pa_oracle.c) — TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA library:
it compiles and loads its own C source with gcc and takes plain NumPy arrays.

Arrays of 16-bit floats travel as ``uint16`` bit patterns and FP8 as ``uint8``
bytes, with a dtype code (0 f16, 1 bf16, 2 fp8 e4m3, 3 f32) beside them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

F16, BF16, FP8_E4M3, F32 = 0, 1, 2, 3

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libpa_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into oracle/_build/libpa_oracle.so (plain gcc)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-Wall",
             "-Wextra", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _SO)
    return _SO


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    lib.or_f16_to_double.argtypes = [ctypes.c_uint16]
    lib.or_f16_to_double.restype = ctypes.c_double
    lib.or_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.or_bf16_to_double.restype = ctypes.c_double
    lib.or_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.or_e4m3_to_double.restype = ctypes.c_double
    lib.or_e4m3_from_float.argtypes = [ctypes.c_float]
    lib.or_e4m3_from_float.restype = ctypes.c_uint8
    lib.oracle_reshape_and_cache.argtypes = [
        P, P, ctypes.c_int, i64, i64, P, P, P, i32, i32, i32, i32, ctypes.c_int, P, P]
    lib.oracle_reshape_and_cache.restype = ctypes.c_int
    lib.oracle_paged_attention.argtypes = [
        P, P, P, ctypes.c_int, i32, i32, i32, P, P, P, P, i32, i32, i32, i32,
        ctypes.c_int, P, P, P, i32, ctypes.c_double, P, P, i64, ctypes.c_int]
    lib.oracle_paged_attention.restype = ctypes.c_int
    lib.oracle_paged_attention_ex.argtypes = lib.oracle_paged_attention.argtypes + [
        ctypes.c_int32, P]
    lib.oracle_paged_attention_ex.restype = ctypes.c_int
    lib.oracle_copy_blocks.argtypes = [P, P, P, P, i64, i64, i64, P, i64]
    lib.oracle_copy_blocks.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


class _Bound:
    """The module's functions bound to another build of the oracle source
    (used by the tests that plant a mistake in a copy of the C file)."""

    def __init__(self, so_path):
        self._lib = _bind(ctypes.CDLL(so_path))

    def __getattr__(self, name):
        fn = globals()[name]

        def call(*a, **kw):
            global _lib
            saved, _lib = _lib, self._lib
            try:
                return fn(*a, **kw)
            finally:
                _lib = saved
        return call


def compile_variant(src_path: str, so_path: str):
    """Compile a modified copy of the oracle source and bind it."""
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-o",
                           so_path, src_path, "-lm", "-lpthread"])
    return _Bound(so_path)


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# --- element codecs ---------------------------------------------------------

def f16_to_double(bits: int) -> float:
    return _load().or_f16_to_double(bits)


def bf16_to_double(bits: int) -> float:
    return _load().or_bf16_to_double(bits)


def e4m3_to_double(byte: int) -> float:
    return _load().or_e4m3_to_double(byte)


def e4m3_from_float(x: float) -> int:
    return _load().or_e4m3_from_float(x)


# --- cache write ------------------------------------------------------------

def reshape_and_cache(key, value, src_dtype, slot_mapping, k_cache, v_cache, block_size,
                      kv_dtype, k_scale=None, v_scale=None, token_stride=None):
    """Scatter key/value rows [T, Hkv, D] into k_cache/v_cache in place.

    k_cache, v_cache: [NB, Hkv, BS, D] arrays (uint16 bits, or uint8 for FP8).
    """
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    T = key.shape[0]
    nb, hkv, bs, d = k_cache.shape
    assert bs == block_size
    if token_stride is None:
        key = np.ascontiguousarray(key)
        value = np.ascontiguousarray(value)
        token_stride = hkv * d
    slots = _c(slot_mapping, np.int64)
    ks, vs = _c(k_scale, np.float32), _c(v_scale, np.float32)
    rc = _load().oracle_reshape_and_cache(
        _ptr(key), _ptr(value), src_dtype, T, token_stride, _ptr(slots), _ptr(k_cache),
        _ptr(v_cache), nb, bs, hkv, d, kv_dtype, _ptr(ks), _ptr(vs))
    if rc != 0:
        raise ValueError(f"oracle_reshape_and_cache failed: {rc}")


# --- attention --------------------------------------------------------------

def paged_attention(q, q_dtype, cu_seqlens_q, seqlens_k, k_cache, v_cache, kv_dtype,
                    block_tables, scale, k_scale=None, v_scale=None, pairs=None,
                    with_lse=False, num_threads=1, window=0, alibi_slopes=None):
    """fp64 attention over the paged cache.

    q: [total_q, Hq, D] (bit patterns).  pairs: optional (rows, heads) arrays;
    then the result is [num_pairs, D], else [total_q, Hq, D].
    """
    q = np.ascontiguousarray(q)
    total_q, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d == d2
    cu = _c(cu_seqlens_q, np.int32)
    sk = _c(seqlens_k, np.int32)
    bt = _c(block_tables, np.int32)
    if bt.ndim == 1:
        bt = bt.reshape(len(sk), -1)
    ks, vs = _c(k_scale, np.float32), _c(v_scale, np.float32)
    if pairs is None:
        out = np.empty((total_q, hq, d), np.float64)
        lse = np.empty((total_q, hq), np.float64) if with_lse else None
        prow = phead = None
        npairs = 0
    else:
        prow = _c(pairs[0], np.int64)
        phead = _c(pairs[1], np.int32)
        npairs = len(prow)
        out = np.empty((npairs, d), np.float64)
        lse = np.empty((npairs,), np.float64) if with_lse else None
    slopes = _c(alibi_slopes, np.float32)
    rc = _load().oracle_paged_attention_ex(
        _ptr(out), _ptr(lse), _ptr(q), q_dtype, total_q, len(sk), hq, _ptr(cu), _ptr(sk),
        _ptr(np.ascontiguousarray(k_cache)), _ptr(np.ascontiguousarray(v_cache)), nb, bs, hkv, d,
        kv_dtype, _ptr(ks), _ptr(vs), _ptr(bt), bt.shape[1], float(scale), _ptr(prow),
        _ptr(phead), npairs, int(num_threads), int(window), _ptr(slopes))
    if rc != 0:
        raise ValueError(f"oracle_paged_attention failed: {rc}")
    return (out, lse) if with_lse else out


def paged_decode(q, q_dtype, context_lens, k_cache, v_cache, kv_dtype, block_tables, scale,
                 **kw):
    """Decode: one query row per sequence (q_len 1, kv_len = context_lens)."""
    b = len(context_lens)
    cu = np.arange(b + 1, dtype=np.int32)
    return paged_attention(q, q_dtype, cu, context_lens, k_cache, v_cache, kv_dtype,
                           block_tables, scale, **kw)


# --- whole-block copies ---------------------------------------------------------

def copy_blocks(dst_k, dst_v, src_k, src_v, pairs):
    """Block dst of dst_k/dst_v takes block src of src_k/src_v for each
    (src, dst) row of pairs; pools are [NB, Hkv, BS, D] arrays (in place)."""
    pairs = _c(np.asarray(pairs).reshape(-1, 2), np.int64)
    bb = int(np.prod(src_k.shape[1:])) * src_k.itemsize
    assert dst_k.flags.c_contiguous and src_k.flags.c_contiguous
    rc = _load().oracle_copy_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v),
                                    src_k.shape[0], dst_k.shape[0], bb, _ptr(pairs), len(pairs))
    if rc != 0:
        raise ValueError(f"oracle_copy_blocks failed: {rc}")
