"""Reference block allocator -- TEST INFRASTRUCTURE ONLY (see oracle/__init__).

What it models (sanketn26 "PagedAttention -- grow the allocation with the
sequence", sections "Separate logical order from physical location", "Sharing
needs ownership rules", "Exercise and checkpoint"; paweldubiel.com
"PagedAttention", "Mechanism and details"; mbrenndoerfer.com "Paged Attention >
Summary", bullets 2 and 4):

* memory is cut into fixed-size physical blocks of ``block_size`` token
  positions; a sequence's block table maps logical block n to a physical block;
* a new block is taken only when a token lands on a block boundary
  (position p with p % block_size == 0), never by moving the prefix;
* position p lives in slot ``table[p // bs] * bs + p % bs``;
* forked sequences share the parent's blocks (refcount + 1 each);
* a shared block is copied before it is written (copy-on-write);
* finishing a sequence releases each block nobody else references.

Where the pages leave the policy open, this model fixes it (the CUDA-side C++
allocator must match it bit for bit):

* the free list is a FIFO queue initialised with ``free_order`` (identity by
  default); blocks are taken from the head and returned to the tail;
* copy-on-write is decided once, at the first token of an append: if the last
  block is partially filled and its refcount is above 1, the appending
  sequence takes a fresh block (popped before any new block of the same
  append), the pair (old, new) is reported, and the old block's refcount drops
  by one; the last remaining owner writes in place;
* a freed sequence releases its blocks in ascending logical order;
* an append that would need more free blocks than exist, or more table
  entries than ``max_blocks_per_seq`` (when non-zero), fails and changes
  nothing.
"""
from __future__ import annotations

from collections import deque
from typing import Dict, List, Optional, Sequence, Tuple


class AllocError(Exception):
    code = -1


class InvalidArg(AllocError):
    code = -1


class OutOfBlocks(AllocError):
    code = -3


class UnknownSeq(AllocError):
    code = -4


class SeqTooLong(AllocError):
    code = -7


class RefAllocator:
    def __init__(self, num_blocks: int, block_size: int,
                 free_order: Optional[Sequence[int]] = None, max_blocks_per_seq: int = 0):
        if num_blocks <= 0 or block_size <= 0 or max_blocks_per_seq < 0:
            raise InvalidArg("bad sizes")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise InvalidArg("free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.bs = block_size
        self.max_blocks = max_blocks_per_seq
        self.free: deque = deque(order)
        self.ref: List[int] = [0] * num_blocks
        self.tables: Dict[int, List[int]] = {}
        self.lens: Dict[int, int] = {}

    # -- sequence lifecycle -------------------------------------------------
    def add(self, sid: int) -> None:
        if sid in self.tables:
            raise InvalidArg(f"sequence {sid} exists")
        self.tables[sid] = []
        self.lens[sid] = 0

    def _seq(self, sid: int) -> List[int]:
        if sid not in self.tables:
            raise UnknownSeq(f"unknown sequence {sid}")
        return self.tables[sid]

    def append(self, sid: int, n: int) -> Tuple[List[int], Optional[Tuple[int, int]]]:
        """Reserve slots for positions len..len+n-1; returns (slots, cow_pair)."""
        table = self._seq(sid)
        if n < 0:
            raise InvalidArg("negative token count")
        if n == 0:
            return [], None
        L = self.lens[sid]
        bs = self.bs
        blocks_before = -(-L // bs)
        blocks_after = -(-(L + n) // bs)
        cow = L % bs != 0 and self.ref[table[-1]] > 1
        need = (blocks_after - blocks_before) + (1 if cow else 0)
        if self.max_blocks and blocks_after > self.max_blocks:
            raise SeqTooLong(f"sequence {sid} would need {blocks_after} blocks")
        if need > len(self.free):
            raise OutOfBlocks(f"need {need} blocks, {len(self.free)} free")
        pair = None
        if cow:
            old = table[-1]
            new = self.free.popleft()
            self.ref[old] -= 1
            self.ref[new] = 1
            table[-1] = new
            pair = (old, new)
        slots = []
        for p in range(L, L + n):
            if p % bs == 0:
                b = self.free.popleft()
                self.ref[b] = 1
                table.append(b)
            slots.append(table[p // bs] * bs + p % bs)
        self.lens[sid] = L + n
        return slots, pair

    def fork(self, parent: int, child: int) -> None:
        table = self._seq(parent)
        if child in self.tables:
            raise InvalidArg(f"sequence {child} exists")
        for b in table:
            self.ref[b] += 1
        self.tables[child] = list(table)
        self.lens[child] = self.lens[parent]

    def free_seq(self, sid: int) -> None:
        table = self._seq(sid)
        for b in table:
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.tables[sid]
        del self.lens[sid]

    # -- views --------------------------------------------------------------
    def table(self, sid: int) -> List[int]:
        return list(self._seq(sid))

    def length(self, sid: int) -> int:
        self._seq(sid)
        return self.lens[sid]

    def free_list(self) -> List[int]:
        return list(self.free)

    def stats(self) -> dict:
        used = sum(1 for r in self.ref if r > 0)
        shared = sum(1 for r in self.ref if r > 1)
        entries = sum(len(t) for t in self.tables.values())
        tokens = sum(self.lens.values())
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": len(self.free),
            "used_blocks": used,
            "shared_blocks": shared,
            "num_seqs": len(self.tables),
            "table_entries": entries,
            "logical_tokens": tokens,
            "reserved_slots": used * self.bs,
        }
