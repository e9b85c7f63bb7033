"""Independent NumPy fp64 twin of the C oracle — TEST INFRASTRUCTURE ONLY.

Used only to cross-check ``pa_oracle.c``: it restates the same definitions
("PagedAttention 与 Continuous Batching", §3.3 data structure and §3.6 kernel;
the V1 packed step of "推理优化与服务：从 PagedAttention 到分离式部署") with
vectorised NumPy in place of scalar C loops, and decodes/encodes the element
formats by different routes (NumPy's IEEE half type, a sorted table of all
E4M3 values searched for the nearest neighbour).
"""
from __future__ import annotations

import numpy as np

F16, BF16, FP8_E4M3, F32 = 0, 1, 2, 3


def to_f64(bits: np.ndarray, dtype: int) -> np.ndarray:
    bits = np.asarray(bits)
    if dtype == F16:
        return bits.astype(np.uint16).view(np.float16).astype(np.float64)
    if dtype == BF16:
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == F32:
        return bits.astype(np.float32).astype(np.float64)
    if dtype == FP8_E4M3:
        return e4m3_decode(bits)
    raise ValueError(dtype)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return s * mag


_POS_CODES = np.arange(0x7F, dtype=np.uint8)           # 0x00 .. 0x7E, finite
_POS_VALUES = e4m3_decode(_POS_CODES)                   # strictly increasing


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 value, ties to the even code, saturating at 448."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    hi = np.clip(np.searchsorted(_POS_VALUES, a, side="left"), 1, len(_POS_VALUES) - 1)
    lo = hi - 1
    dlo = a - _POS_VALUES[lo]
    dhi = _POS_VALUES[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (_POS_CODES[hi] % 2 == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo]).astype(np.uint8)
    code = np.where(a >= 448.0, np.uint8(0x7E), code)
    code = np.where(np.signbit(x), code | np.uint8(0x80), code)
    code = np.where(np.isnan(x), np.uint8(0x7F), code)
    return code.astype(np.uint8)


def reshape_and_cache(key, value, src_dtype, slot_mapping, k_cache, v_cache, kv_dtype,
                      k_scale=None, v_scale=None):
    nb, hkv, bs, d = k_cache.shape
    slots = np.asarray(slot_mapping, np.int64)
    keep = slots >= 0
    blk, off = slots[keep] // bs, slots[keep] % bs
    if kv_dtype == FP8_E4M3:
        ks = np.asarray(k_scale, np.float32).astype(np.float64)[None, :, None]
        vs = np.asarray(v_scale, np.float32).astype(np.float64)[None, :, None]
        kq = (to_f64(key[keep], src_dtype) / ks).astype(np.float32)
        vq = (to_f64(value[keep], src_dtype) / vs).astype(np.float32)
        k_cache[blk, :, off, :] = e4m3_encode(kq)
        v_cache[blk, :, off, :] = e4m3_encode(vq)
    else:
        k_cache[blk, :, off, :] = key[keep]
        v_cache[blk, :, off, :] = value[keep]


def paged_attention(q, q_dtype, cu_seqlens_q, seqlens_k, k_cache, v_cache, kv_dtype,
                    block_tables, scale, k_scale=None, v_scale=None):
    total_q, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    g = hq // hkv
    qf = to_f64(q, q_dtype)
    out = np.zeros((total_q, hq, d), np.float64)
    bt = np.asarray(block_tables).reshape(len(seqlens_k), -1)
    for r in range(len(seqlens_k)):
        r0, r1 = int(cu_seqlens_q[r]), int(cu_seqlens_q[r + 1])
        q_len, kv_len = r1 - r0, int(seqlens_k[r])
        if kv_len == 0 or q_len == 0:
            continue
        t = np.arange(kv_len)
        blk, off = bt[r, t // bs], t % bs
        kc = to_f64(k_cache[blk, :, off, :], kv_dtype)      # [kv_len, Hkv, D]
        vc = to_f64(v_cache[blk, :, off, :], kv_dtype)
        if kv_dtype == FP8_E4M3:
            kc = kc * np.asarray(k_scale, np.float32).astype(np.float64)[None, :, None]
            vc = vc * np.asarray(v_scale, np.float32).astype(np.float64)[None, :, None]
        kh = np.repeat(kc, g, axis=1)                         # [kv_len, Hq, D]
        vh = np.repeat(vc, g, axis=1)
        rows = np.arange(q_len)
        last = kv_len - q_len + rows                          # inclusive
        mask = t[None, :] <= last[:, None]                    # [q_len, kv_len]
        s = float(scale) * np.einsum("ihd,thd->hit", qf[r0:r1], kh)
        s = np.where(mask[None], s, -np.inf)
        m = s.max(axis=-1, keepdims=True)
        live = np.isfinite(m)
        w = np.where(live, np.exp(s - np.where(live, m, 0.0)), 0.0)
        den = w.sum(axis=-1, keepdims=True)
        o = np.einsum("hit,thd->ihd", w, vh) / np.where(den > 0, den, 1.0).transpose(1, 0, 2)
        out[r0:r1] = o
    return out
