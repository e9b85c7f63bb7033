"""Seeded synthetic inputs for the paged-attention path.

This module only draws inputs: random values, sequence lengths, block
allocations, block tables and slot mappings, the way a continuous-batching
scheduler would hand them to the attention step ("PagedAttention 与 Continuous
Batching", §2.5 step 4 builds token ids, block_tables and slot_mapping; §3.3
data structure).  It holds none of the attention arithmetic, so both the CUDA
path and the CPU oracle can be fed from it.

Conventions (shared by every consumer):
  * 16-bit floats are returned as ``uint16`` bit patterns (bf16 or IEEE f16),
    drawn in fp32 from N(0, 1) and rounded to nearest even.
  * The KV pool is ``[num_blocks, num_kv_heads, block_size, head_dim]``; a
    token at logical position t of a sequence with table ``bt`` lives at slot
    ``bt[t // block_size] * block_size + t % block_size``.
  * Table entries past ``ceil(len / block_size)`` are -1 and must never be read.
  * ``prefill_*``: tokens already cached before the step (written to the pool
    once, outside any timed region).  ``new_*``: the step's own tokens, written
    by reshape_and_cache in the step, in packed query-row order.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

F16, BF16, FP8_E4M3, F32 = 0, 1, 2, 3
DTYPE_NAMES = {F16: "f16", BF16: "bf16", FP8_E4M3: "fp8_e4m3", F32: "f32"}
BLOCK_SIZE = 16
_CHUNK = 1 << 24


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bfloat16 (nearest even); inputs here are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bits_to_f32(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Widen bf16/f16 bit patterns to fp32 (exact)."""
    if dtype == BF16:
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float32)
    raise ValueError(dtype)


def _round_into(out: np.ndarray, x: np.ndarray, dtype: int) -> None:
    """out[:] = x rounded to the 16-bit format (nearest even), in place on x."""
    if dtype == BF16:
        u = x.view(np.uint32)
        t = u >> np.uint32(16)
        t &= np.uint32(1)
        t += np.uint32(0x7FFF)
        t += u
        t >>= np.uint32(16)
        out[:] = t
    else:
        out[:] = x.astype(np.float16).view(np.uint16)


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        import concurrent.futures
        import os
        _POOL = concurrent.futures.ThreadPoolExecutor(max(1, min(8, (os.cpu_count() or 1))))
    return _POOL


def randn_bits(rng: np.random.Generator, shape, dtype: int) -> np.ndarray:
    """N(0,1) samples rounded to a 16-bit float format, drawn in chunks.

    The draws are sequential (one stream from ``rng``); the rounding of each
    chunk runs on a worker thread while the next chunk is drawn."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    jobs = []
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        x = rng.standard_normal(e - s, dtype=np.float32)
        jobs.append(_pool().submit(_round_into, out[s:e], x, dtype))
    for j in jobs:
        j.result()
    return out.reshape(shape)


@dataclasses.dataclass
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    block_size: int
    q_dtype: int
    src_dtype: int            # dtype of the new K/V rows handed to the cache write
    kv_dtype: int             # pool dtype (== src_dtype, or FP8_E4M3)
    out_dtype: int
    scale: float              # fp32 logit scale
    q: np.ndarray             # [total_q, Hq, D] uint16
    cu_seqlens_q: np.ndarray  # [B + 1] int32
    seqlens_k: np.ndarray     # [B] int32, cached + new keys
    block_tables: np.ndarray  # [B, max_blocks_per_seq] int32, -1 padded
    prefill_k: np.ndarray     # [T_pre, Hkv, D] uint16
    prefill_v: np.ndarray
    prefill_slots: np.ndarray  # [T_pre] int64
    new_k: np.ndarray         # [total_q, Hkv, D] uint16
    new_v: np.ndarray
    new_slots: np.ndarray     # [total_q] int64, -1 = nothing to write
    k_scale: Optional[np.ndarray] = None   # [Hkv] float32 (FP8 only)
    v_scale: Optional[np.ndarray] = None
    partition_size: int = 0
    decode: bool = True       # every request has q_len 1

    @property
    def total_q(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def q_lens(self) -> np.ndarray:
        return np.diff(self.cu_seqlens_q).astype(np.int32)

    @property
    def context_lens(self) -> np.ndarray:
        return self.seqlens_k

    @property
    def max_context_len(self) -> int:
        return int(self.seqlens_k.max()) if len(self.seqlens_k) else 0

    @property
    def max_q_len(self) -> int:
        return int(self.q_lens.max()) if len(self.seqlens_k) else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    def kv_elem_bytes(self) -> int:
        return 1 if self.kv_dtype == FP8_E4M3 else 2

    def kv_bytes_read(self) -> int:
        """Bytes of K and V that attention must read: every visible key of
        every (request, KV head) once (query heads of a GQA group share it)."""
        per_tok = 2 * self.num_kv_heads * self.head_dim * self.kv_elem_bytes()
        return int(self.seqlens_k.astype(np.int64).sum()) * per_tok

    def unique_kv_bytes_read(self) -> int:
        """Bytes of distinct physical slots attention touches (shared blocks once)."""
        bs = self.block_size
        slots = set()
        toks = 0
        for r in range(self.num_seqs):
            L = int(self.seqlens_k[r])
            for i in range(-(-L // bs)):
                b = int(self.block_tables[r, i])
                n = min(bs, L - i * bs)
                if b in slots:
                    continue
                slots.add(b)
                toks += n
        per_tok = 2 * self.num_kv_heads * self.head_dim * self.kv_elem_bytes()
        return toks * per_tok


def _slots_for(table: np.ndarray, positions: np.ndarray, bs: int) -> np.ndarray:
    return table[positions // bs].astype(np.int64) * bs + positions % bs


def build_workload(name: str, seed: int, q_lens: Sequence[int], kv_lens: Sequence[int],
                   num_q_heads: int, num_kv_heads: int, head_dim: int, dtype: int = BF16,
                   kv_dtype: Optional[int] = None, out_dtype: Optional[int] = None,
                   num_blocks: Optional[int] = None, alloc: str = "permutation",
                   shared_prefix_len: int = 0, pool_slack: float = 1.1,
                   extra_table_cols: int = 1, partition_size: int = 0,
                   block_size: int = BLOCK_SIZE) -> Workload:
    """Draw one step's inputs.

    q_lens[r] query rows of request r attend its kv_lens[r] keys; the last
    q_lens[r] of those keys are the step's new tokens.  Blocks are handed out
    from a seeded random permutation of the pool (alloc='permutation') or as a
    seeded random choice of distinct ids (alloc='choice').  With
    shared_prefix_len = P (a multiple of the block size), logical blocks
    0 .. P/bs - 1 of every request are the same physical blocks, and the prefix
    tokens are written once.
    """
    rng = np.random.default_rng(seed)
    kv_dtype = dtype if kv_dtype is None else kv_dtype
    out_dtype = dtype if out_dtype is None else out_dtype
    q_lens = np.asarray(q_lens, np.int64)
    kv_lens = np.asarray(kv_lens, np.int64)
    B = len(kv_lens)
    bs = block_size
    assert len(q_lens) == B and np.all(q_lens <= kv_lens) and np.all(q_lens >= 0)
    assert shared_prefix_len % bs == 0
    n_shared = shared_prefix_len // bs
    need = -(-kv_lens // bs)                               # blocks per request
    if n_shared:
        assert np.all(kv_lens >= shared_prefix_len)
    private = need - n_shared
    total_blocks = int(n_shared + private.sum())
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(pool_slack * total_blocks)))
    assert num_blocks >= total_blocks, "pool too small"
    if alloc == "permutation":
        ids = rng.permutation(num_blocks)[:total_blocks]
    elif alloc == "choice":
        ids = rng.choice(num_blocks, total_blocks, replace=False)
    else:
        raise ValueError(alloc)
    ids = ids.astype(np.int32)
    width = int(need.max() if B else 0) + extra_table_cols
    tables = np.full((B, max(width, 1)), -1, np.int32)
    shared_ids = ids[:n_shared]
    cursor = n_shared
    for r in range(B):
        tables[r, :n_shared] = shared_ids
        k = int(private[r])
        tables[r, n_shared:n_shared + k] = ids[cursor:cursor + k]
        cursor += k

    Hkv, D = num_kv_heads, head_dim
    src = BF16 if kv_dtype == FP8_E4M3 and dtype not in (BF16, F16) else dtype
    # cached context: shared prefix once, then every request's private part
    pre_pos: List[np.ndarray] = []
    pre_slots: List[np.ndarray] = []
    if n_shared:
        p = np.arange(shared_prefix_len)
        pre_slots.append(_slots_for(tables[0], p, bs))
    for r in range(B):
        lo = shared_prefix_len if n_shared else 0
        hi = int(kv_lens[r] - q_lens[r])
        if hi > lo:
            p = np.arange(lo, hi)
            pre_slots.append(_slots_for(tables[r], p, bs))
    prefill_slots = (np.concatenate(pre_slots) if pre_slots else np.zeros(0, np.int64))
    new_slots_l = []
    for r in range(B):
        p = np.arange(int(kv_lens[r] - q_lens[r]), int(kv_lens[r]))
        s = _slots_for(tables[r], p, bs)
        if n_shared:
            s = np.where(p < shared_prefix_len, -1, s)   # already cached, shared
        new_slots_l.append(s)
    new_slots = (np.concatenate(new_slots_l) if new_slots_l else np.zeros(0, np.int64))
    total_q = int(q_lens.sum())

    prefill_k = randn_bits(rng, (len(prefill_slots), Hkv, D), src)
    prefill_v = randn_bits(rng, (len(prefill_slots), Hkv, D), src)
    new_k = randn_bits(rng, (total_q, Hkv, D), src)
    new_v = randn_bits(rng, (total_q, Hkv, D), src)
    q = randn_bits(rng, (total_q, num_q_heads, D), dtype if dtype != FP8_E4M3 else BF16)

    k_scale = v_scale = None
    if kv_dtype == FP8_E4M3:
        # one scale per KV head, max|x| / 448 over that head's data, so no
        # value saturates
        def head_absmax(a, b):
            m = np.zeros(Hkv, np.float32)
            for arr in (a, b):
                for s in range(0, arr.shape[0], 1 << 16):
                    blk = np.abs(bits_to_f32(arr[s:s + (1 << 16)], src))
                    if blk.size:
                        m = np.maximum(m, blk.max(axis=(0, 2)))
            return m
        k_scale = (head_absmax(prefill_k, new_k) / np.float32(448.0)).astype(np.float32)
        v_scale = (head_absmax(prefill_v, new_v) / np.float32(448.0)).astype(np.float32)
        k_scale[k_scale == 0] = 1.0
        v_scale[v_scale == 0] = 1.0

    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum(q_lens)
    return Workload(
        name=name, num_seqs=B, num_q_heads=num_q_heads, num_kv_heads=Hkv, head_dim=D,
        num_blocks=int(num_blocks), block_size=bs,
        q_dtype=(dtype if dtype != FP8_E4M3 else BF16), src_dtype=src, kv_dtype=kv_dtype,
        out_dtype=out_dtype, scale=float(np.float32(1.0 / math.sqrt(D))), q=q,
        cu_seqlens_q=cu, seqlens_k=kv_lens.astype(np.int32), block_tables=tables,
        prefill_k=prefill_k, prefill_v=prefill_v, prefill_slots=prefill_slots,
        new_k=new_k, new_v=new_v, new_slots=new_slots, k_scale=k_scale, v_scale=v_scale,
        partition_size=partition_size, decode=bool(np.all(q_lens == 1)))


# --------------------------------------------------------------------------
# The five reference workloads
# --------------------------------------------------------------------------

CONFIG_NAMES = {
    1: "tiny MHA paged decode (B 4, L {1,17,40,100}, 2/2 heads, D 64, f16)",
    2: "LLaMA-13B-shaped MHA decode (B 64, L U[128,2048], 40/40 heads, D 128, bf16)",
    3: "Llama-3-8B-shaped GQA decode (B 256, L lognormal median 1000 in [32,8192], 32/8, D 128, bf16)",
    4: "mixed continuous-batching step (200 decodes + 4x512 chunks, 32/8, D 128, bf16)",
    5: "shared-prefix long-context decode (B 128, 2048 shared + U[0,6144], 32/8, D 128, FP8 KV)",
}


def config(i: int, seed: Optional[int] = None, batch: Optional[int] = None) -> Workload:
    """Reference workload i (1..5), seeded with 1000 + i unless given.

    ``batch`` shrinks the request count (same distributions) for tests.
    """
    seed = 1000 + i if seed is None else seed
    rng = np.random.default_rng(seed + 7919)
    if i == 1:
        lens = np.array([1, 17, 40, 100])
        return build_workload("config1_tiny_mha", seed, np.ones(4, np.int64), lens, 2, 2, 64,
                              dtype=F16, num_blocks=64, alloc="choice")
    if i == 2:
        B = 64 if batch is None else batch
        lens = rng.integers(128, 2048, size=B, endpoint=True)
        return build_workload("config2_llama13b_mha", seed, np.ones(B, np.int64), lens, 40, 40,
                              128, dtype=BF16, num_blocks=12000)
    if i == 3:
        B = 256 if batch is None else batch
        lens = np.clip(np.rint(rng.lognormal(math.log(1000.0), 1.0, size=B)), 32, 8192)
        return build_workload("config3_llama3_8b_gqa", seed, np.ones(B, np.int64),
                              lens.astype(np.int64), 32, 8, 128, dtype=BF16, partition_size=512)
    if i == 4:
        nd = 200 if batch is None else batch
        c = rng.integers(64, 4096, size=nd, endpoint=True)
        prior = np.array([0, 1024, 2048, 3072])
        q_lens = np.concatenate([np.ones(nd, np.int64), np.full(4, 512)])
        kv_lens = np.concatenate([c + 1, prior + 512])
        return build_workload("config4_mixed_step", seed, q_lens, kv_lens, 32, 8, 128,
                              dtype=BF16)
    if i == 5:
        B = 128 if batch is None else batch
        suffix = rng.integers(0, 6144, size=B, endpoint=True)
        lens = 2048 + suffix
        return build_workload("config5_shared_prefix_fp8", seed, np.ones(B, np.int64), lens, 32,
                              8, 128, dtype=BF16, kv_dtype=FP8_E4M3, out_dtype=BF16,
                              shared_prefix_len=2048)
    raise ValueError(i)

