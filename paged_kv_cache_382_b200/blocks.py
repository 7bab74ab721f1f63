"""Host-side KV block manager: free list, reference counts, per-sequence block
tables, lazy allocation and copy-on-write planning.

This is the bookkeeping that decides *where* K/V live; the device kernels only
follow its output (``block_tables``, ``slot_mapping``, copy pairs).  It does no
attention arithmetic.

Behaviour, after the pages:
  * A sequence's tokens fill logical blocks of ``block_size`` tokens; each
    logical block is mapped to a physical block of the shared pool through the
    sequence's block table ("PagedAttention blog", section 3(3); "Month 2 ·
    PagedAttention", section 02 mapping table).
  * A new physical block is taken only when a token crosses into the next
    logical block -- lazy allocation, the counterpart of a page fault
    ("Month 2 · PagedAttention", section 02).
  * Forked sequences (parallel samples of one prompt) share the prompt's
    physical blocks; each physical block counts its sharers ("PagedAttention
    blog", section 4, step 1).
  * A sharer that writes into a physical block whose count is above one gets a
    fresh block holding a copy of the old one, and the old block's count drops
    by one; the last remaining sharer writes in place ("PagedAttention blog",
    section 4, step 2).
  * Slot of token position ``pos``: ``table[pos // B] * B + pos % B`` (reading
    adopted; the pages only say the K/V are filled into the physical blocks
    through the mapping).
"""

from __future__ import annotations

from collections import deque
from dataclasses import dataclass, field
from typing import Iterable, List, Optional, Tuple

import numpy as np


class OutOfBlocks(RuntimeError):
    """The free list is empty."""


class BlockPool:
    """Physical blocks ``0 .. num_blocks-1`` with a free list and ref counts."""

    def __init__(self, num_blocks: int, free_order: Optional[Iterable[int]] = None):
        self.num_blocks = int(num_blocks)
        order = list(range(self.num_blocks)) if free_order is None else [int(b) for b in free_order]
        if len(set(order)) != len(order) or any(b < 0 or b >= self.num_blocks for b in order):
            raise ValueError("free_order must list distinct block ids in [0, num_blocks)")
        self.ref_cnt = np.zeros(self.num_blocks, dtype=np.int64)
        self._free = deque(order)

    @property
    def num_free(self) -> int:
        return len(self._free)

    def allocate(self) -> int:
        if not self._free:
            raise OutOfBlocks(
                f"failed to allocate a block: all {self.num_blocks} blocks of the pool are in use")
        block = self._free.popleft()
        self.ref_cnt[block] = 1
        return block

    def incref(self, block: int) -> None:
        if self.ref_cnt[block] <= 0:
            raise ValueError(f"block {block} is free")
        self.ref_cnt[block] += 1

    def decref(self, block: int) -> None:
        if self.ref_cnt[block] <= 0:
            raise ValueError(f"block {block} is already free")
        self.ref_cnt[block] -= 1
        if self.ref_cnt[block] == 0:
            self._free.append(block)


@dataclass
class Sequence:
    """One request's view: its block table and how many tokens it holds."""

    block_table: List[int] = field(default_factory=list)
    num_tokens: int = 0

    def filled(self, block_size: int) -> List[int]:
        """Number of filled slots of each logical block (the '# filled' column)."""
        return [min(block_size, self.num_tokens - i * block_size) for i in range(len(self.block_table))]


class BlockManager:
    """Allocates slots for appended tokens and plans copy-on-write copies."""

    def __init__(self, pool: BlockPool, block_size: int):
        if block_size <= 0:
            raise ValueError("block_size must be positive")
        self.pool = pool
        self.block_size = int(block_size)

    def new_sequence(self) -> Sequence:
        return Sequence()

    def append_tokens(self, seq: Sequence, n: int) -> Tuple[List[int], List[Tuple[int, int]]]:
        """Reserve slots for ``n`` new tokens of ``seq``.

        Returns (slots, copies): the slot of each new token in order, and the
        (src, dst) block copies that must run before those writes.
        """
        slots: List[int] = []
        copies: List[Tuple[int, int]] = []
        B = self.block_size
        for _ in range(int(n)):
            pos = seq.num_tokens
            logical = pos // B
            if logical == len(seq.block_table):
                seq.block_table.append(self.pool.allocate())
            else:
                physical = seq.block_table[logical]
                if self.pool.ref_cnt[physical] > 1:
                    fresh = self.pool.allocate()
                    copies.append((physical, fresh))
                    self.pool.decref(physical)
                    seq.block_table[logical] = fresh
            slots.append(seq.block_table[logical] * B + pos % B)
            seq.num_tokens += 1
        return slots, copies

    def fork(self, seq: Sequence) -> Sequence:
        """A new sequence sharing every physical block of ``seq``."""
        for block in seq.block_table:
            self.pool.incref(block)
        return Sequence(block_table=list(seq.block_table), num_tokens=seq.num_tokens)

    def free(self, seq: Sequence) -> None:
        # last block first: under least-recently-freed reuse a shared prefix stays longest
        for block in reversed(seq.block_table):
            self.pool.decref(block)
        seq.block_table = []
        seq.num_tokens = 0


def block_table_array(seqs: List[Sequence], max_blocks: Optional[int] = None, fill: int = -1) -> np.ndarray:
    """Pack block tables into an int32 [num_seqs][max_blocks] array; unused entries = ``fill``."""
    width = max((len(s.block_table) for s in seqs), default=0) if max_blocks is None else int(max_blocks)
    width = max(width, 1)
    out = np.full((len(seqs), width), fill, dtype=np.int32)
    for i, s in enumerate(seqs):
        if len(s.block_table) > width:
            raise ValueError("max_blocks is smaller than a block table")
        out[i, : len(s.block_table)] = s.block_table
    return out
