"""Host-side model of the KV block manager the pages describe.

TEST INFRASTRUCTURE ONLY (it builds expected block tables, slots and
copy-on-write pairs for the tests; the product's kernels only ever see block
tables, slots and copy pairs).

Behaviour, with the passage each rule follows:
  * Fixed-size blocks, a per-sequence block table mapping logical block i to
    a physical block, blocks allocated one at a time as the sequence grows:
    "PagedAttention and KV memory management" (introduction) and "How does
    vLLM PagedAttention manage Virtual Memory Pages ...", sections "Detail"
    and "Key Technical Innovations" (items 1 and 2).
  * The free list starts as every block id in increasing order and is used
    first-in first-out (the same page, section "Example").  Freed blocks
    return to the tail; the pages do not say where they go.
  * A new block is taken when the token being appended is the first of a
    logical block, i.e. when its position pos (0-based, equal to the length
    before the append) satisfies pos % block_size == 0.  For block_size > 1
    this is the page's "length after the append is 1 mod block_size" rule;
    unlike that rule it also fires for block_size == 1.
  * Reference counts and copy-on-write: "Paged Attention: OS-Inspired Memory
    Management for KV Caches", section "Key terms in this lesson" (Reference
    count; Copy-on-write).  A fork points the child at the parent's blocks
    and raises their counts; a write into a block whose count is above one
    first moves the writer onto a private copy (returned as a (src, dst)
    pair for copy_blocks); the last sharer writes in place.
  * The slot of position pos is table[pos // block_size] * block_size +
    pos % block_size.
"""
from __future__ import annotations

from collections import deque


class OutOfBlocks(RuntimeError):
    """Raised when an allocation finds the free list empty."""


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(range(num_blocks))
        self.refcount = [0] * num_blocks
        self.tables: dict[object, list[int]] = {}
        self.lengths: dict[object, int] = {}

    # -- allocation ---------------------------------------------------------
    def _take(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free KV block left")
        blk = self.free.popleft()
        assert self.refcount[blk] == 0
        self.refcount[blk] = 1
        return blk

    def _release(self, blk: int) -> None:
        assert self.refcount[blk] > 0
        self.refcount[blk] -= 1
        if self.refcount[blk] == 0:
            self.free.append(blk)

    # -- sequences ----------------------------------------------------------
    def add_sequence(self, seq) -> None:
        if seq in self.tables:
            raise KeyError(f"sequence {seq!r} exists")
        self.tables[seq] = []
        self.lengths[seq] = 0

    def append_token(self, seq):
        """Reserve the slot of the next token of seq.

        Returns (slot, cow_pairs): cow_pairs lists the (src, dst) block copies
        that must run before the token is written.
        """
        if seq not in self.tables:
            self.add_sequence(seq)
        table = self.tables[seq]
        pos = self.lengths[seq]
        bs = self.block_size
        pairs = []
        if pos % bs == 0:
            table.append(self._take())
        else:
            last = table[-1]
            if self.refcount[last] > 1:
                fresh = self._take()
                self.refcount[last] -= 1
                table[-1] = fresh
                pairs.append((last, fresh))
        self.lengths[seq] = pos + 1
        return self.slot(seq, pos), pairs

    def fork(self, parent, child) -> None:
        """child shares every block of parent (reference counts go up)."""
        if child in self.tables:
            raise KeyError(f"sequence {child!r} exists")
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for blk in self.tables[child]:
            self.refcount[blk] += 1

    def free_sequence(self, seq) -> None:
        for blk in self.tables.pop(seq):
            self._release(blk)
        del self.lengths[seq]

    # -- queries ------------------------------------------------------------
    def slot(self, seq, pos: int) -> int:
        table = self.tables[seq]
        return table[pos // self.block_size] * self.block_size + pos % self.block_size

    def block_table(self, seq) -> list[int]:
        return list(self.tables[seq])

    def num_free(self) -> int:
        return len(self.free)
