"""Oracle block manager: the host-side bookkeeping of a paged KV cache, in
plain Python.

TEST INFRASTRUCTURE ONLY (see ``oracle.paged_kv``): the library's C++ block
manager is checked against this class, decision for decision.

Sources:

* [LSHU] lshu.cn/news/11644, vLLM architecture analysis.
  - "整体架构": one global physical pool; a request gets blocks on demand when
    it arrives and gives them back the moment it finishes; no reservation.
  - "方案：页式内存管理": fixed-size blocks, one Block Table per request, a free
    block pool; a request that grows by one token writes into its last block
    if that block still has room, otherwise takes a block from the pool and
    appends its index to the table; a finished request returns all of its
    blocks to the pool.
  - "收益分析": any free block can serve any request (no external
    fragmentation); "内存共享": requests with the same prefix share the same
    physical blocks read-only, and a later divergence is handled by
    copy-on-write.

Readings where the pages are silent (each is a choice, applied identically by
the C++ manager):

* the free pool is a first-in first-out queue, initially blocks 0 .. N-1 in
  order; blocks whose last reference goes away join its tail in table order;
* a block is shared when its reference count (number of Block Tables that
  hold it) is above one; appending into a shared, non-full last block first
  copies it into a fresh block (the copy pair is reported, the old block loses
  one reference) and then writes into the copy;
* one decode step appends one token to each listed sequence, in list order,
  and is all-or-nothing: if the pool cannot supply every block the step needs,
  nothing changes.
"""

from __future__ import annotations

from collections import deque


class OutOfBlocks(RuntimeError):
    pass


class BlockManager:
    """Free pool, reference counts and one Block Table per sequence."""

    def __init__(self, num_blocks: int, block_size: int, max_blocks_per_seq: int, free_order=None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_blocks_per_seq = max_blocks_per_seq
        self.free = deque(range(num_blocks) if free_order is None else free_order)
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    # -- allocation ---------------------------------------------------------
    def _take(self) -> int:
        if not self.free:
            raise OutOfBlocks
        b = self.free.popleft()
        self.ref[b] = 1
        return b

    def _release(self, b: int) -> None:
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    # -- requests -----------------------------------------------------------
    def add_sequence(self, seq_id: int, num_tokens: int) -> list[int]:
        """A new request with ``num_tokens`` prompt tokens: blocks for all of
        them, taken from the pool; returns the prompt tokens' slots."""
        if seq_id in self.tables:
            raise KeyError(seq_id)
        B = self.block_size
        nb = -(-num_tokens // B)
        if nb > self.max_blocks_per_seq:
            raise ValueError("sequence longer than the Block Table")
        if nb > len(self.free):
            raise OutOfBlocks
        table = [self._take() for _ in range(nb)]
        self.tables[seq_id] = table
        self.lens[seq_id] = num_tokens
        return [table[t // B] * B + t % B for t in range(num_tokens)]

    def fork(self, parent: int, child: int) -> None:
        """``child`` starts as ``parent``: same tokens, same physical blocks."""
        if child in self.tables or parent not in self.tables:
            raise KeyError(child)
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def blocks_needed(self, seq_ids) -> int:
        """Blocks that ``append`` of one token to each listed sequence takes:
        one per full (or missing) last block, one per copy.  Of k listed
        owners of one shared block with r references, min(k, r - 1) copy it."""
        n = 0
        B = self.block_size
        copied: dict[int, int] = {}
        for s in seq_ids:
            L = self.lens[s]
            if L % B == 0:
                n += 1
                continue
            last = self.tables[s][-1]
            if self.ref[last] - copied.get(last, 0) > 1:
                copied[last] = copied.get(last, 0) + 1
                n += 1
        return n

    def append(self, seq_ids) -> tuple[list[int], list[tuple[int, int]]]:
        """One decode step: one new token per listed sequence.  Returns the
        new tokens' slots and the (src, dst) block copies to run first."""
        seq_ids = list(seq_ids)
        if len(set(seq_ids)) != len(seq_ids) or any(s not in self.tables for s in seq_ids):
            raise KeyError(seq_ids)
        B = self.block_size
        for s in seq_ids:
            if self.lens[s] % B == 0 and len(self.tables[s]) + 1 > self.max_blocks_per_seq:
                raise ValueError("sequence longer than the Block Table")
        # Count before changing anything.  A block that loses a reference to a
        # copy is still held by another table, so no block is freed mid-step.
        if self.blocks_needed(seq_ids) > len(self.free):
            raise OutOfBlocks
        slots, copies = [], []
        for s in seq_ids:
            table, L = self.tables[s], self.lens[s]
            if L % B == 0:
                table.append(self._take())
            elif self.ref[table[-1]] > 1:
                old = table[-1]
                new = self._take()
                self.ref[old] -= 1
                table[-1] = new
                copies.append((old, new))
            slots.append(table[-1] * B + L % B)
            self.lens[s] = L + 1
        return slots, copies

    def free_sequence(self, seq_id: int) -> None:
        """A finished request gives back its blocks at once."""
        for b in self.tables.pop(seq_id):
            self._release(b)
        del self.lens[seq_id]

    # -- views --------------------------------------------------------------
    def block_tables(self, seq_ids) -> tuple[list[list[int]], list[int]]:
        """Block Table rows padded with -1 to ``max_blocks_per_seq``, and the
        context lengths, of the listed sequences."""
        rows = []
        for s in seq_ids:
            t = self.tables[s]
            rows.append(t + [-1] * (self.max_blocks_per_seq - len(t)))
        return rows, [self.lens[s] for s in seq_ids]
