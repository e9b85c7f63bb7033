"""Python binding of libpa (ctypes): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it turns torch tensors into device pointers, sizes and
dtype codes, runs the call on the one device its tensors sit on with that
device's current CUDA stream (or the stream given), and raises
:class:`PaError` on a non-zero status.  The library must be built in-tree
(``python -m paged_kv_cache_lens_b200.build``); importing this module without
it raises, so there is no silent CPU fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "pa.h")

PA_F16, PA_BF16, PA_FP8_E4M3, PA_F32 = 0, 1, 2, 3
PA_OK = 0
STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED",
                3: "PA_ERR_WORKSPACE", 4: "PA_ERR_OUT_OF_RANGE", 5: "PA_ERR_CUDA",
                6: "PA_ERR_TIMEOUT"}


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {pa_status_string(status)}")


class pa_attn_options(ctypes.Structure):
    _fields_ = [("window", ctypes.c_int32), ("alibi_slopes", ctypes.c_void_p)]


class pa_cache_desc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int), ("k_scale", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libpa.so and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m paged_kv_cache_lens_b200.build`")
    lib = ctypes.CDLL(path)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    E, F = ctypes.c_int, ctypes.c_float
    D = ctypes.POINTER(pa_cache_desc)
    lib.pa_status_string.argtypes = [E]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_reshape_and_cache.argtypes = [P, P, E, i64, i64, P, P, P, D, P]
    lib.pa_reshape_and_cache.restype = E
    lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.pa_decode_workspace_size.restype = sz
    lib.pa_decode.argtypes = [P, E, P, E, i32, i32, P, P, D, P, i32, P, i32, F, i32, P, sz, P]
    lib.pa_decode.restype = E
    lib.pa_varlen_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.pa_varlen_workspace_size.restype = sz
    lib.pa_varlen_workspace_size_ex.argtypes = [i32, i32, i32, i32, i32, i32, i32, E, E]
    lib.pa_varlen_workspace_size_ex.restype = sz
    lib.pa_varlen.argtypes = [P, E, P, E, i32, i32, i32, P, P, i32, i32, P, P, D, P, i32, F, P,
                              sz, P]
    lib.pa_varlen.restype = E
    lib.pa_device_error.argtypes = [P]
    lib.pa_device_error.restype = E
    O = ctypes.POINTER(pa_attn_options)
    lib.pa_decode_ex.argtypes = [P, E, P, E, i32, i32, P, P, D, P, i32, P, i32, F, i32, O, P, sz,
                                 P]
    lib.pa_decode_ex.restype = E
    lib.pa_varlen_ex.argtypes = [P, E, P, E, i32, i32, i32, P, P, i32, i32, P, P, D, P, i32, F, O,
                                 P, sz, P]
    lib.pa_varlen_ex.restype = E
    lib.pa_copy_blocks.argtypes = [P, P, D, P, i64, P]
    lib.pa_copy_blocks.restype = E
    lib.pa_swap_blocks.argtypes = [P, P, P, P, D, i64, i64, P, i64, P]
    lib.pa_swap_blocks.restype = E
    lib.pa_selftest_wait_timeout.argtypes = [P]
    lib.pa_selftest_wait_timeout.restype = E
    lib.pa_hbm_read_probe.argtypes = [P, i64, P, P]
    lib.pa_hbm_read_probe.restype = E
    if path == LIB_PATH:
        _lib = lib
    return lib


def declared_functions(header: str = HEADER):
    """Names of the entry points include/pa.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


# --------------------------------------------------------------------------
# marshalling helpers
# --------------------------------------------------------------------------

def dtype_code(t: torch.dtype, fp8_if_byte: bool = False) -> int:
    if t == torch.float16:
        return PA_F16
    if t == torch.bfloat16:
        return PA_BF16
    if t == torch.float32:
        return PA_F32
    if t in (torch.uint8, getattr(torch, "float8_e4m3fn", None)):
        return PA_FP8_E4M3
    raise ValueError(f"no libpa dtype for {t}")


def _need(t: Optional[torch.Tensor], name: str, dtype=None, rows_strided: bool = False,
          pinned_ok: bool = False) -> None:
    """The library reads every tensor through a raw pointer with a fixed
    layout: reject, before any launch, what it would misread (a host tensor,
    a non-contiguous view, the wrong element type)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if rows_strided:
        # [rows, ...] with any row stride, each row itself contiguous
        if t.dim() < 2 or (t.shape[0] > 0 and not t[0].is_contiguous()):
            raise ValueError(f"{name}: each row must be contiguous")
    elif not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.device.type != "cuda" and not (pinned_ok and t.is_pinned()):
        where = "CUDA or pinned host memory" if pinned_ok else "a CUDA tensor"
        raise ValueError(f"{name}: must be {where} (got {t.device})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _device_of(*tensors) -> Optional[torch.device]:
    """The one CUDA device the call's device tensors sit on (None and pinned
    host tensors are skipped; None when no tensor is on a device).  The
    library launches on the current device and dereferences every pointer
    there, so tensors on two devices are refused before the call."""
    dev = None
    for t in tensors:
        if t is None or t.device.type != "cuda":
            continue
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on {dev} and {t.device}: a call takes one CUDA device")
    return dev


def _on(dev: Optional[torch.device]):
    """Make `dev` the current device for the call (nothing to do for None)."""
    return torch.cuda.device(dev) if dev is not None else contextlib.nullcontext()


def _stream(stream, dev: Optional[torch.device] = None) -> ctypes.c_void_p:
    """The stream handle: the given stream, else the current stream of `dev`
    (of the current device when `dev` is None).  A torch stream of another
    device than the tensors' is refused."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    if isinstance(stream, torch.cuda.Stream):
        if dev is not None and stream.device != dev:
            raise ValueError(f"stream of {stream.device} for tensors on {dev}")
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def cache_desc(k_cache: torch.Tensor, k_scale=None, v_scale=None) -> pa_cache_desc:
    nb, hkv, bs, d = k_cache.shape
    return pa_cache_desc(nb, bs, hkv, d, dtype_code(k_cache.dtype), _ptr(k_scale).value
                         if k_scale is not None else None,
                         _ptr(v_scale).value if v_scale is not None else None)


def _check(status: int, where: str):
    if status != PA_OK:
        raise PaError(status, where)


# --------------------------------------------------------------------------
# entry points
# --------------------------------------------------------------------------

def pa_status_string(status: int) -> str:
    try:
        return load_library().pa_status_string(int(status)).decode()
    except ImportError:
        return STATUS_NAMES.get(int(status), "PA_ERR_UNKNOWN")


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, slot_mapping: torch.Tensor,
                         k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale=None,
                         v_scale=None, stream=None) -> None:
    """key/value: [T, Hkv, D] (rows may be strided, e.g. views into a fused QKV
    buffer); slot_mapping: int64 [T]; pools [NB, Hkv, block_size, D]."""
    _need(key, "key", rows_strided=True)
    _need(value, "value", rows_strided=True)
    if key.shape != value.shape or key.stride() != value.stride():
        raise ValueError("key and value must have the same shape and strides")
    _need(slot_mapping, "slot_mapping", torch.int64)
    _need(k_cache, "k_cache")
    _need(v_cache, "v_cache")
    _need(k_scale, "k_scale", torch.float32)
    _need(v_scale, "v_scale", torch.float32)
    dev = _device_of(key, value, slot_mapping, k_cache, v_cache, k_scale, v_scale)
    T = key.shape[0]
    desc = cache_desc(k_cache, k_scale, v_scale)
    with _on(dev):
        st = load_library().pa_reshape_and_cache(
            _ptr(key), _ptr(value), dtype_code(key.dtype), T, key.stride(0) if T else 0,
            _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache), ctypes.byref(desc),
            _stream(stream, dev))
    _check(st, "pa_reshape_and_cache")


def pa_decode_workspace_size(batch: int, num_q_heads: int, head_dim: int, max_context_len: int,
                             partition_size: int = 0) -> int:
    return int(load_library().pa_decode_workspace_size(batch, num_q_heads, head_dim,
                                                       max_context_len, partition_size))


def pa_varlen_workspace_size(num_seqs: int, total_q: int, num_q_heads: int, head_dim: int,
                             max_context_len: int) -> int:
    return int(load_library().pa_varlen_workspace_size(num_seqs, total_q, num_q_heads, head_dim,
                                                       max_context_len))


def pa_varlen_workspace_size_ex(num_seqs: int, total_q: int, num_q_heads: int,
                                num_kv_heads: int, head_dim: int, max_q_len: int,
                                max_context_len: int, q_dtype: int, kv_dtype: int) -> int:
    """Workspace for exactly these sizes and dtype codes (PA_F16 / PA_BF16 /
    PA_FP8_E4M3): split-K partials only for the rows the decode kernel runs."""
    return int(load_library().pa_varlen_workspace_size_ex(
        num_seqs, total_q, num_q_heads, num_kv_heads, head_dim, max_q_len, max_context_len,
        q_dtype, kv_dtype))


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]):
    if nbytes == 0:
        return workspace, 0 if workspace is None else workspace.numel()
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def _options(window: int, alibi_slopes: Optional[torch.Tensor]):
    if not window and alibi_slopes is None:
        return None
    return ctypes.byref(pa_attn_options(int(window or 0), _ptr(alibi_slopes).value
                                        if alibi_slopes is not None else None))


def pa_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int,
              scale: float, k_scale=None, v_scale=None, partition_size: int = 0,
              workspace: Optional[torch.Tensor] = None, stream=None, window: int = 0,
              alibi_slopes: Optional[torch.Tensor] = None) -> None:
    """out/q: [B, Hq, D]; block_tables int32 [B, max_blocks]; context_lens int32 [B].
    window / alibi_slopes select pa_decode_ex's sliding window and ALiBi."""
    for t, n in ((out, "out"), (q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (workspace, "workspace")):
        _need(t, n)
    _need(block_tables, "block_tables", torch.int32)
    _need(context_lens, "context_lens", torch.int32)
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale"), (alibi_slopes, "alibi_slopes")):
        _need(t, n, torch.float32)
    dev = _device_of(out, q, k_cache, v_cache, workspace, block_tables, context_lens, k_scale,
                     v_scale, alibi_slopes)
    B, hq, d = q.shape
    lib = load_library()
    need = lib.pa_decode_workspace_size(B, hq, d, max_context_len, partition_size)
    workspace, wbytes = _workspace(need, q.device, workspace)
    desc = cache_desc(k_cache, k_scale, v_scale)
    args = (_ptr(out), dtype_code(out.dtype), _ptr(q), dtype_code(q.dtype), B, hq,
            _ptr(k_cache), _ptr(v_cache), ctypes.byref(desc), _ptr(block_tables),
            block_tables.shape[1], _ptr(context_lens), int(max_context_len), float(scale),
            int(partition_size))
    opts = _options(window, alibi_slopes)
    with _on(dev):
        if opts is None:
            st = lib.pa_decode(*args, _ptr(workspace), wbytes, _stream(stream, dev))
        else:
            st = lib.pa_decode_ex(*args, opts, _ptr(workspace), wbytes, _stream(stream, dev))
    _check(st, "pa_decode" if opts is None else "pa_decode_ex")


def pa_varlen(out: torch.Tensor, q: torch.Tensor, cu_seqlens_q: torch.Tensor,
              seqlens_k: torch.Tensor, max_q_len: int, max_context_len: int,
              k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
              scale: float, k_scale=None, v_scale=None, workspace: Optional[torch.Tensor] = None,
              stream=None, window: int = 0, alibi_slopes: Optional[torch.Tensor] = None) -> None:
    """out/q: [total_q, Hq, D]; cu_seqlens_q int32 [S+1]; seqlens_k int32 [S].
    window / alibi_slopes select pa_varlen_ex's sliding window and ALiBi."""
    for t, n in ((out, "out"), (q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (workspace, "workspace")):
        _need(t, n)
    for t, n in ((cu_seqlens_q, "cu_seqlens_q"), (seqlens_k, "seqlens_k"),
                 (block_tables, "block_tables")):
        _need(t, n, torch.int32)
    for t, n in ((k_scale, "k_scale"), (v_scale, "v_scale"), (alibi_slopes, "alibi_slopes")):
        _need(t, n, torch.float32)
    dev = _device_of(out, q, k_cache, v_cache, workspace, cu_seqlens_q, seqlens_k, block_tables,
                     k_scale, v_scale, alibi_slopes)
    total_q, hq, d = q.shape
    S = seqlens_k.shape[0]
    lib = load_library()
    need = lib.pa_varlen_workspace_size_ex(S, total_q, hq, k_cache.shape[1], d, int(max_q_len),
                                           max_context_len, dtype_code(q.dtype),
                                           dtype_code(k_cache.dtype))
    if out.data_ptr() % 16:
        need = lib.pa_varlen_workspace_size(S, total_q, hq, d, max_context_len)
    workspace, wbytes = _workspace(need, q.device, workspace)
    desc = cache_desc(k_cache, k_scale, v_scale)
    args = (_ptr(out), dtype_code(out.dtype), _ptr(q), dtype_code(q.dtype), total_q, S, hq,
            _ptr(cu_seqlens_q), _ptr(seqlens_k), int(max_q_len), int(max_context_len),
            _ptr(k_cache), _ptr(v_cache), ctypes.byref(desc), _ptr(block_tables),
            block_tables.shape[1], float(scale))
    opts = _options(window, alibi_slopes)
    with _on(dev):
        if opts is None:
            st = lib.pa_varlen(*args, _ptr(workspace), wbytes, _stream(stream, dev))
        else:
            st = lib.pa_varlen_ex(*args, opts, _ptr(workspace), wbytes, _stream(stream, dev))
    _check(st, "pa_varlen" if opts is None else "pa_varlen_ex")


def pa_hbm_read_probe(buf: torch.Tensor, sink: torch.Tensor, stream=None) -> None:
    """Stream `buf` (contiguous, device) once with read-only loads; sink (a
    device int32 of one element) receives the XOR of its 32-bit words."""
    _need(buf, "buf")
    _need(sink, "sink")
    dev = _device_of(buf, sink)
    with _on(dev):
        st = load_library().pa_hbm_read_probe(_ptr(buf), buf.numel() * buf.element_size(),
                                              _ptr(sink), _stream(stream, dev))
    _check(st, "pa_hbm_read_probe")


def pa_selftest_wait_timeout(stream=None) -> None:
    """Enqueue the library's bounded-wait self-test: the next pa_device_error
    returns PA_ERR_TIMEOUT (6)."""
    _check(load_library().pa_selftest_wait_timeout(_stream(stream)), "pa_selftest_wait_timeout")


def pa_device_error(stream=None) -> int:
    """Read and clear the library's device error word (synchronises the stream)."""
    return int(load_library().pa_device_error(_stream(stream)))


def pa_copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_mapping: torch.Tensor,
                   stream=None) -> None:
    """block_mapping: device int64 [n, 2] of (src, dst) block ids."""
    _need(k_cache, "k_cache")
    _need(v_cache, "v_cache")
    _need(block_mapping, "block_mapping", torch.int64)
    dev = _device_of(k_cache, v_cache, block_mapping)
    desc = cache_desc(k_cache)
    n = block_mapping.shape[0]
    with _on(dev):
        st = load_library().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), ctypes.byref(desc),
                                           _ptr(block_mapping), n, _stream(stream, dev))
    _check(st, "pa_copy_blocks")


def pa_swap_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                   src_v: torch.Tensor, block_mapping, stream=None) -> None:
    """Pools on the device or in pinned host memory; block_mapping: host
    (src, dst) pairs (anything numpy can turn into int64 [n, 2])."""
    import numpy as np
    for t, n in ((dst_k, "dst_k"), (dst_v, "dst_v"), (src_k, "src_k"), (src_v, "src_v")):
        _need(t, n, pinned_ok=True)
    dev = _device_of(dst_k, dst_v, src_k, src_v)
    pairs = np.ascontiguousarray(np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2))
    desc = cache_desc(src_k)
    with _on(dev):
        st = load_library().pa_swap_blocks(
            _ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v), ctypes.byref(desc),
            src_k.shape[0], dst_k.shape[0], ctypes.c_void_p(pairs.ctypes.data), len(pairs),
            _stream(stream, dev))
    _check(st, "pa_swap_blocks")
