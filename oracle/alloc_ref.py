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

Prefix caching (paweldubiel.com "PagedAttention", "Text order is not a memory
address": block sharing is useful for prefix caching; sanketn26 "Use a runtime
that owns the blocks": prefix reuse in a paged runtime).  The pages give no
mechanism; this model fixes one:

* a full block whose token ids are known is indexed under the key
  (physical block of the preceding tokens or -1, its token ids); it enters the
  index when an append with token ids fills it, unless the key is taken;
* a new sequence with token ids takes the longest chain of indexed blocks
  matching its leading full blocks (refcount + 1; a matched block waiting in
  the free list leaves it) and starts with those tokens in place;
* released blocks stay indexed in the free list; a block taken from the free
  list for new use leaves the index.

Swap (sanketn26 "What this does not solve": admission can cause preemption):
a host pool with its own FIFO free list (identity order); swapping a sequence
out moves each table entry, in logical order, to the next host block and
releases the device block; swapping in takes device blocks from the free list
and returns the host blocks to the host free list's tail.
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
        self.tracked: Dict[int, bool] = {}
        self.tokens: Dict[int, List[int]] = {}
        self.index: Dict[Tuple[int, Tuple[int, ...]], int] = {}
        self.key_of: Dict[int, Tuple[int, Tuple[int, ...]]] = {}
        self.hit_blocks = self.query_blocks = self.evicted = 0
        self.host_blocks = 0
        self.host_free: deque = deque()
        self.swapped: Dict[int, List[int]] = {}

    # -- sequence lifecycle -------------------------------------------------
    def add(self, sid: int) -> None:
        if sid in self.tables:
            raise InvalidArg(f"sequence {sid} exists")
        self.tables[sid] = []
        self.lens[sid] = 0
        self.tracked[sid] = False
        self.tokens[sid] = []

    def _seq(self, sid: int) -> List[int]:
        if sid not in self.tables:
            raise UnknownSeq(f"unknown sequence {sid}")
        return self.tables[sid]

    def _live(self, sid: int) -> List[int]:
        table = self._seq(sid)
        if sid in self.swapped:
            raise InvalidArg(f"sequence {sid} is swapped out")
        return table

    def _take(self) -> int:
        """Head of the free list for new use; it leaves the prefix index."""
        b = self.free.popleft()
        if b in self.key_of:
            del self.index[self.key_of.pop(b)]
            self.evicted += 1
        return b

    def _release(self, b: int) -> None:
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def append(self, sid: int, n: int) -> Tuple[List[int], Optional[Tuple[int, int]]]:
        """Reserve slots for positions len..len+n-1; returns (slots, cow_pair).
        The sequence's token ids are unknown afterwards."""
        res = self._append(sid, n)
        if n > 0:
            self.tracked[sid] = False
        return res

    def _append(self, sid: int, n: int) -> Tuple[List[int], Optional[Tuple[int, int]]]:
        table = self._live(sid)
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
            new = self._take()
            self.ref[old] -= 1
            self.ref[new] = 1
            table[-1] = new
            pair = (old, new)
        slots = []
        for p in range(L, L + n):
            if p % bs == 0:
                b = self._take()
                self.ref[b] = 1
                table.append(b)
            slots.append(table[p // bs] * bs + p % bs)
        self.lens[sid] = L + n
        return slots, pair

    def fork(self, parent: int, child: int) -> None:
        table = self._live(parent)
        if child in self.tables:
            raise InvalidArg(f"sequence {child} exists")
        for b in table:
            self.ref[b] += 1
        self.tables[child] = list(table)
        self.lens[child] = self.lens[parent]
        self.tracked[child] = self.tracked[parent]
        self.tokens[child] = list(self.tokens[parent])

    def free_seq(self, sid: int) -> None:
        table = self._seq(sid)
        if sid in self.swapped:
            self.host_free.extend(self.swapped.pop(sid))
        else:
            for b in table:
                self._release(b)
        for d in (self.tables, self.lens, self.tracked, self.tokens):
            del d[sid]

    # -- prefix caching -------------------------------------------------------
    def add_cached(self, sid: int, token_ids: Sequence[int]) -> int:
        """New sequence sharing the longest indexed chain of full blocks that
        matches its leading tokens; returns the number of tokens in place."""
        if sid in self.tables:
            raise InvalidArg(f"sequence {sid} exists")
        toks = [int(t) for t in token_ids]
        bs = self.bs
        full = len(toks) // bs
        if self.max_blocks:
            full = min(full, self.max_blocks)
        table: List[int] = []
        for j in range(full):
            key = (table[-1] if table else -1, tuple(toks[j * bs:(j + 1) * bs]))
            b = self.index.get(key)
            if b is None:
                break
            if self.ref[b] == 0:
                self.free.remove(b)
            self.ref[b] += 1
            table.append(b)
        self.hit_blocks += len(table)
        self.query_blocks += full
        self.tables[sid] = table
        self.lens[sid] = len(table) * bs
        self.tracked[sid] = True
        self.tokens[sid] = toks[:len(table) * bs]
        return len(table) * bs

    def append_tokens(self, sid: int, token_ids: Sequence[int]
                      ) -> Tuple[List[int], Optional[Tuple[int, int]]]:
        """append() for a sequence with known token ids; blocks it fills enter
        the index (unless their key is taken)."""
        self._live(sid)
        if not self.tracked[sid]:
            raise InvalidArg(f"sequence {sid} has no token history")
        toks = [int(t) for t in token_ids]
        L = self.lens[sid]
        res = self._append(sid, len(toks))
        self.tokens[sid] += toks
        table, bs = self.tables[sid], self.bs
        for j in range(L // bs, self.lens[sid] // bs):
            key = (table[j - 1] if j > 0 else -1, tuple(self.tokens[sid][j * bs:(j + 1) * bs]))
            b = table[j]
            if b in self.key_of or key in self.index:
                continue
            self.index[key] = b
            self.key_of[b] = key
        return res

    # -- swap ---------------------------------------------------------------
    def set_host_pool(self, n: int) -> None:
        if self.swapped:
            raise InvalidArg("host pool in use")
        self.host_blocks = n
        self.host_free = deque(range(n))

    def swap_out(self, sid: int) -> List[Tuple[int, int]]:
        table = self._live(sid)
        if len(table) > len(self.host_free):
            raise OutOfBlocks("host pool short")
        pairs, host = [], []
        for b in table:
            h = self.host_free.popleft()
            pairs.append((b, h))
            host.append(h)
            self._release(b)
        self.tables[sid] = []
        self.swapped[sid] = host
        return pairs

    def swap_in(self, sid: int) -> List[Tuple[int, int]]:
        self._seq(sid)
        if sid not in self.swapped:
            raise InvalidArg(f"sequence {sid} is not swapped out")
        host = self.swapped[sid]
        if len(host) > len(self.free):
            raise OutOfBlocks("device pool short")
        pairs, table = [], []
        for h in host:
            b = self._take()
            self.ref[b] = 1
            table.append(b)
            pairs.append((h, b))
            self.host_free.append(h)
        del self.swapped[sid]
        self.tables[sid] = table
        return pairs

    # -- views --------------------------------------------------------------
    def table(self, sid: int) -> List[int]:
        t = self._seq(sid)
        return list(self.swapped[sid]) if sid in self.swapped else list(t)

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
            "cached_blocks": len(self.index),
            "prefix_hit_blocks": self.hit_blocks,
            "prefix_query_blocks": self.query_blocks,
            "evicted_blocks": self.evicted,
            "host_blocks": self.host_blocks,
            "host_free_blocks": len(self.host_free),
            "swapped_seqs": len(self.swapped),
        }
