"""Host-side block bookkeeping: allocation, reference counts, fork and
copy-on-write ("PagedAttention 与 Continuous Batching", §3.2-§3.3 free pool and
block tables; §3.8 COW 与引用计数).

The manager decides *which* slot each new token goes to and *which* blocks
must be copied; the device work is done by the library (pa_reshape_and_cache
writes the slots, pa_copy_blocks performs the copies it schedules).
"""
from __future__ import annotations

from collections import deque
from typing import Dict, Iterable, List, Optional, Tuple


class OutOfBlocks(RuntimeError):
    pass


class BlockManager:
    """Every call either completes or raises with the pool unchanged: a table
    that does not fit takes no block, and a release of a block nobody holds is
    refused rather than corrupting the counts."""

    def __init__(self, num_blocks: int, block_size: int = 16,
                 free_order: Optional[Iterable[int]] = None):
        if num_blocks < 0 or block_size < 1:
            raise ValueError("num_blocks must be >= 0 and block_size >= 1")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if len(set(order)) != len(order) or any(not 0 <= b < num_blocks for b in order):
            raise ValueError("free_order must hold distinct block ids in [0, num_blocks)")
        self.free: deque = deque(order)
        self.ref: Dict[int, int] = {}

    # -- pool -----------------------------------------------------------------
    def allocate(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free block")
        b = self.free.popleft()
        self.ref[b] = 1
        return b

    def release(self, block: int) -> None:
        if self.ref.get(block, 0) < 1:
            raise ValueError(f"block {block} is not held by any sequence")
        self.ref[block] -= 1
        if self.ref[block] == 0:
            del self.ref[block]
            self.free.append(block)

    def free_table(self, table: List[int]) -> None:
        """A finished sequence returns every block it references."""
        self._check_held(table)
        for b in table:
            self.release(b)

    def _check_held(self, table: List[int]) -> None:
        """Every block of the table is held at least as often as it appears."""
        for b in set(table):
            if self.ref.get(b, 0) < table.count(b):
                raise ValueError(f"block {b} is not held by this table")

    def ref_count(self, block: int) -> int:
        return self.ref.get(block, 0)

    # -- sequences ----------------------------------------------------------------
    def allocate_table(self, num_tokens: int) -> List[int]:
        """Blocks for a new sequence of num_tokens tokens, all or none."""
        if num_tokens < 0:
            raise ValueError("num_tokens must be >= 0")
        n = -(-num_tokens // self.block_size)
        if n > len(self.free):
            raise OutOfBlocks(f"{n} blocks needed, {len(self.free)} free")
        return [self.allocate() for _ in range(n)]

    def fork(self, table: List[int], n: int) -> List[List[int]]:
        """n sequences sharing the parent's blocks (parallel sampling / beam
        search): every shared block's reference count grows by n - 1."""
        if n < 1:
            raise ValueError("a fork makes at least one sequence")
        self._check_held(table)
        for b in table:
            self.ref[b] += n - 1
        return [list(table) for _ in range(n)]

    def append_slot(self, table: List[int], num_tokens: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Slot for token index num_tokens (the sequence holds num_tokens tokens).

        A full last block gets a fresh block appended; a last block that other
        sequences still reference (ref_count > 1) is copied first: a new block
        is allocated, the (src, dst) copy is returned for pa_copy_blocks, the
        table is redirected and the shared block loses one reference.
        Returns (slot, copy or None); the table is updated in place.
        """
        bs = self.block_size
        idx, off = divmod(num_tokens, bs)
        if num_tokens < 0 or idx > len(table) or (idx == len(table) and off != 0):
            raise ValueError(f"token {num_tokens} does not follow a table of {len(table)} blocks")
        copy = None
        if idx == len(table):
            table.append(self.allocate())
        elif self.ref[table[idx]] > 1:
            src = table[idx]
            dst = self.allocate()
            self.release(src)
            table[idx] = dst
            copy = (src, dst)
        return table[idx] * bs + off, copy
