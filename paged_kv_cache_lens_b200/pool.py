"""KV pool sizing arithmetic ("PagedAttention 与 Continuous Batching", §8.3
KV 显存测算 and exercise 2 of §10.7)."""
from __future__ import annotations


def kv_bytes_per_block(block_size: int, num_layers: int, num_kv_heads: int, head_dim: int,
                       dtype_bytes: int) -> int:
    """Bytes one physical block occupies across all layers, K and V together."""
    return block_size * 2 * num_layers * num_kv_heads * head_dim * dtype_bytes


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int,
                       dtype_bytes: int) -> int:
    return 2 * num_layers * num_kv_heads * head_dim * dtype_bytes


def max_concurrent_sequences(kv_budget_bytes: int, avg_context: int, num_layers: int,
                             num_kv_heads: int, head_dim: int, dtype_bytes: int,
                             block_size: int = 16) -> int:
    """How many sequences of avg_context tokens fit a KV budget, counting whole
    blocks per sequence."""
    blocks_per_seq = -(-avg_context // block_size)
    per_block = kv_bytes_per_block(block_size, num_layers, num_kv_heads, head_dim, dtype_bytes)
    return kv_budget_bytes // (blocks_per_seq * per_block)
