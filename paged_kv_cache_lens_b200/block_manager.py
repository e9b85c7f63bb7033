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
    def __init__(self, num_blocks: int, block_size: int = 16,
                 free_order: Optional[Iterable[int]] = None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free: deque = deque(range(num_blocks) if free_order is None else free_order)
        self.ref: Dict[int, int] = {}

    # -- pool -----------------------------------------------------------------
    def allocate(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free block")
        b = self.free.popleft()
        self.ref[b] = 1
        return b

    def release(self, block: int) -> None:
        self.ref[block] -= 1
        if self.ref[block] == 0:
            del self.ref[block]
            self.free.append(block)

    def free_table(self, table: List[int]) -> None:
        """A finished sequence returns every block it references."""
        for b in table:
            self.release(b)

    def ref_count(self, block: int) -> int:
        return self.ref.get(block, 0)

    # -- sequences ----------------------------------------------------------------
    def allocate_table(self, num_tokens: int) -> List[int]:
        return [self.allocate() for _ in range(-(-num_tokens // self.block_size))]

    def fork(self, table: List[int], n: int) -> List[List[int]]:
        """n sequences sharing the parent's blocks (parallel sampling / beam
        search): every shared block's reference count grows by n - 1."""
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
