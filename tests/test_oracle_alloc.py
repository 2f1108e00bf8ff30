"""Pins for the reference allocator (oracle/alloc_ref.py) against the numbers
the pages print and the invariants they state."""
import math
import random

import numpy as np
import pytest

from conftest import golden
from oracle.alloc_ref import (InvalidArg, OutOfBlocks, RefAllocator, SeqTooLong, UnknownSeq)
import workloads


def _order(first, n):
    rest = [b for b in range(n) if b not in first]
    return list(first) + rest


def test_placement_example():
    g = golden("placement_example.json")
    bs = g["block_size"]
    a = RefAllocator(8, bs, _order(g["physical"], 8))
    a.add(0)
    slots, pair = a.append(0, g["length"])
    assert pair is None
    assert a.table(0) == g["physical"]
    assert len(a.table(0)) == g["blocks"] and len(a.table(0)) * bs == g["slots"]
    used_last = g["length"] - (g["blocks"] - 1) * bs
    assert used_last == g["last_block_used"] and bs - used_last == g["last_block_free"]
    # position p lives at table[p // bs] * bs + p % bs
    assert slots == [4 * 4 + 0, 4 * 4 + 1, 4 * 4 + 2, 4 * 4 + 3, 1 * 4 + 0]


def test_block_diagram_growth():
    g = golden("block_diagram.json")
    bs = g["block_size"]
    a = RefAllocator(16, bs, _order(g["physical"], 16))
    a.add(0)
    a.append(0, g["tokens"])
    assert a.table(0) == g["physical"]
    nfree = len(a.free)
    for p in g["fit_positions"]:
        slots, _ = a.append(0, 1)
        assert slots == [g["physical"][-1] * bs + p % bs]
        assert len(a.free) == nfree, "positions that fit must not take a block"
    slots, _ = a.append(0, 1)
    assert a.length(0) == g["new_block_position"] + 1
    assert len(a.free) == nfree - 1 and len(a.table(0)) == len(g["physical"]) + 1
    assert slots == [a.table(0)[-1] * bs + 0]


def test_capacity_table():
    g = golden("capacity_table.json")
    bs = g["block_size"]
    a = RefAllocator(64, bs)
    for i, L in enumerate(g["lengths"]):
        a.add(i)
        a.append(i, L)
    st = a.stats()
    assert len(g["lengths"]) * g["max_length"] == g["reserve_max_positions"]
    assert st["reserved_slots"] == g["block_positions"]
    assert st["logical_tokens"] == g["occupied_positions"]
    assert g["reserve_max_positions"] - st["reserved_slots"] == g["saved_positions"]
    assert st["reserved_slots"] - st["logical_tokens"] == g["unused_in_final_blocks"]
    # the tiny workload appends one token to each of 5/9/14: 6/10/15 still fit
    before = st["used_blocks"]
    for i in range(3):
        a.append(i, 1)
    assert a.stats()["used_blocks"] == before


def test_growth_exercise_and_release():
    g = golden("growth_exercise.json")
    bs = g["block_size"]
    a = RefAllocator(32, bs)
    a.add(0); a.append(0, g["grow_from"])
    a.add(1); a.append(1, g["finished_length"])
    assert len(a.table(0)) == g["blocks_before"]
    a.append(0, g["grow_to"] - g["grow_from"])
    assert len(a.table(0)) == g["blocks_after"]
    nfree = len(a.free)
    a.free_seq(1)
    assert len(a.free) - nfree == g["released_blocks"]
    # released only when nobody else references them
    a.add(2); a.append(2, g["finished_length"])
    a.fork(2, 3)
    nfree = len(a.free)
    a.free_seq(2)
    assert len(a.free) == nfree
    a.free_seq(3)
    assert len(a.free) - nfree == g["released_blocks"]


def test_free_list_fifo_and_release_order():
    a = RefAllocator(6, 2, [5, 4, 3, 2, 1, 0])
    a.add(0); a.append(0, 5)          # takes 5, 4, 3
    assert a.table(0) == [5, 4, 3]
    a.free_seq(0)                     # returns them in logical order to the tail
    assert a.free_list() == [2, 1, 0, 5, 4, 3]


def test_copy_on_write_rules():
    bs = 4
    a = RefAllocator(32, bs)
    a.add(0); a.append(0, 6)          # blocks 0, 1 (block 1 half full)
    a.fork(0, 1); a.fork(0, 2)
    assert a.ref[1] == 3
    s, pair = a.append(1, 1)          # shared partial block -> private copy
    assert pair == (1, 2) and a.table(1) == [0, 2] and s == [2 * bs + 2]
    assert a.ref[1] == 2 and a.ref[2] == 1
    s, pair = a.append(2, 3)          # copy, then the rest of the block, then a new block
    assert pair == (1, 3) and a.table(2) == [0, 3, 4]
    assert s == [3 * bs + 2, 3 * bs + 3, 4 * bs + 0]
    s, pair = a.append(0, 1)          # last owner writes in place
    assert pair is None and a.table(0) == [0, 1] and s == [1 * bs + 2]
    # a full shared block never needs a copy: the next token opens a new block
    b = RefAllocator(8, bs)
    b.add(0); b.append(0, 8); b.fork(0, 1)
    s, pair = b.append(1, 1)
    assert pair is None and b.table(1)[:2] == b.table(0) and len(b.table(1)) == 3


def test_failures_leave_state_unchanged():
    a = RefAllocator(4, 4, max_blocks_per_seq=3)
    a.add(0); a.append(0, 6)          # blocks 0, 1
    a.fork(0, 1)
    a.add(2); a.append(2, 4)          # block 2; one block left
    snap = (list(a.free), list(a.ref), {k: list(v) for k, v in a.tables.items()}, dict(a.lens))
    with pytest.raises(OutOfBlocks):
        a.append(1, 5)                # 1 copy + 1 new > 1 free
    with pytest.raises(SeqTooLong):
        a.append(0, 7)                # 13 tokens -> 4 blocks > 3
    with pytest.raises(UnknownSeq):
        a.append(9, 1)
    with pytest.raises(UnknownSeq):
        a.free_seq(9)
    with pytest.raises(InvalidArg):
        a.fork(0, 1)
    with pytest.raises(InvalidArg):
        a.add(0)
    with pytest.raises(InvalidArg):
        a.append(0, -1)
    assert snap == (list(a.free), list(a.ref), {k: list(v) for k, v in a.tables.items()},
                    dict(a.lens))
    a.free_seq(1)
    with pytest.raises(UnknownSeq):
        a.free_seq(1)                 # double free
    with pytest.raises(InvalidArg):
        RefAllocator(4, 4, [0, 1, 1, 3])


def _check_invariants(a: RefAllocator):
    bs = a.bs
    free = list(a.free)
    assert len(set(free)) == len(free)
    in_tables = set(b for t in a.tables.values() for b in t)
    assert not (set(free) & in_tables)
    assert len(free) + len(in_tables) == a.num_blocks
    counts = {}
    for t in a.tables.values():
        for b in t:
            counts[b] = counts.get(b, 0) + 1
    assert all(a.ref[b] == c for b, c in counts.items())
    assert sum(a.ref) == sum(len(t) for t in a.tables.values())
    for sid, t in a.tables.items():
        # at most one partially filled block per sequence (mbrenndoerfer.com
        # "Paged Attention > Summary", bullet 2)
        waste = len(t) * bs - a.lens[sid]
        assert 0 <= waste <= bs - 1


@pytest.mark.parametrize("seed", range(6))
def test_random_ops_keep_invariants(seed):
    r = random.Random(seed)
    bs = r.choice([1, 2, 4, 8, 16])
    a = RefAllocator(64, bs, list(np.random.default_rng(seed).permutation(64)))
    live, nxt = [], 0
    for _ in range(400):
        kind = r.random()
        try:
            if kind < 0.15 or not live:
                a.add(nxt); live.append(nxt); nxt += 1
            elif kind < 0.7:
                a.append(r.choice(live), r.choice([0, 1, 1, 1, 2, 5, 17]))
            elif kind < 0.85:
                a.fork(r.choice(live), nxt); live.append(nxt); nxt += 1
            else:
                s = r.choice(live); a.free_seq(s); live.remove(s)
        except OutOfBlocks:
            pass
        _check_invariants(a)


def test_beam_sharing_counts():
    """Config 4 by its event list: closed-form block counts and the >= 50% claim."""
    g = golden("beam_saving.json")
    wl = workloads.beam(steps=256)
    sh = wl.shape
    bs, prefix, groups, beams = sh.block_size, 2050, 4, 4
    a = RefAllocator(sh.num_blocks, bs, sh.free_order)
    steps = 0
    pairs_first = None
    for st in _ops_only(wl):
        npairs = 0
        for op in st:
            if op[0] == "add": a.add(op[1])
            elif op[0] == "fork": a.fork(op[1], op[2])
            elif op[0] == "append":
                _, pair = a.append(op[1], op[2]); npairs += pair is not None
        if steps == 0:
            assert a.stats()["used_blocks"] == groups * math.ceil(prefix / bs)
        if steps == 1:
            pairs_first = npairs
            assert a.stats()["used_blocks"] == groups * (math.ceil(prefix / bs) + (beams - 1))
        steps += 1
    assert pairs_first == groups * (beams - 1)
    final_len = prefix + 256
    shared_full = prefix // bs
    private = math.ceil(final_len / bs) - shared_full
    used = a.stats()["used_blocks"]
    assert used == groups * (shared_full + beams * private) == 784
    unshared = groups * beams * math.ceil(final_len / bs)
    assert unshared == 2320
    assert 1 - used / unshared >= g["min_saving"]


def _ops_only(wl):
    """The event lists of a workload without drawing its values."""
    import itertools
    # the beam generator draws values lazily per step; pull ops step by step
    for st in wl.steps:
        yield st.ops


# ---------------------------------------------------------------- prefix caching
def _tok(n, base=0):
    return list(range(base, base + n))


def test_prefix_blocks_are_shared_and_partial_blocks_are_not():
    bs = 4
    a = RefAllocator(32, bs)
    T = _tok(10)                        # 2 full blocks + 2 tokens
    assert a.add_cached(1, T) == 0      # empty index
    a.append_tokens(1, T)
    assert a.stats()["cached_blocks"] == 2
    # same first 8 tokens, different tail: both full blocks are shared
    assert a.add_cached(2, T[:8] + [99, 98, 97]) == 8
    assert a.table(2) == a.table(1)[:2]
    assert [a.ref[b] for b in a.table(1)[:2]] == [2, 2]
    # diverging inside block 1: only block 0 is shared
    assert a.add_cached(3, T[:5] + [77, 76, 75]) == 4
    assert a.table(3) == a.table(1)[:1] and a.ref[a.table(1)[0]] == 3
    # the same tokens under a different parent block never match
    assert a.add_cached(4, [50, 51, 52, 53] + T[4:8]) == 0
    st = a.stats()
    assert st["prefix_hit_blocks"] == 3 and st["prefix_query_blocks"] == 2 + 2 + 2 + 2


def test_prefix_cache_survives_release_and_is_evicted_in_fifo_order():
    bs = 4
    a = RefAllocator(8, bs, list(range(8)))
    T = _tok(8)
    a.add_cached(1, T)
    a.append_tokens(1, T)               # blocks 0, 1 indexed
    a.free_seq(1)
    assert a.free_list() == [2, 3, 4, 5, 6, 7, 0, 1]
    assert a.stats()["cached_blocks"] == 2
    # a hit takes the cached blocks out of the free list, wherever they are
    assert a.add_cached(2, T + [9]) == 8
    assert a.table(2) == [0, 1] and 0 not in a.free_list() and 1 not in a.free_list()
    assert a.stats()["free_blocks"] == 6
    a.free_seq(2)
    # new allocations walk the FIFO: blocks 2..7 first, then the cached 0 and 1
    a.add(3)
    a.append(3, 6 * bs)
    assert a.stats()["cached_blocks"] == 2 and a.stats()["evicted_blocks"] == 0
    a.append(3, 1)                      # takes block 0: evicted from the index
    st = a.stats()
    assert st["cached_blocks"] == 1 and st["evicted_blocks"] == 1
    # block 1 is still indexed but its parent (block 0) is gone: no chain match
    assert a.add_cached(4, T) == 0


def test_identical_blocks_are_indexed_once():
    bs = 4
    a = RefAllocator(16, bs)
    T = _tok(8)
    a.add_cached(1, T)
    a.append_tokens(1, T)
    assert a.add_cached(2, T[:3]) == 0  # no full block to match
    a.append_tokens(2, T[3:8])          # fills two blocks with seq 1's tokens
    # block 0's key (-1, T[0:4]) is taken, so it is not indexed; block 1's key
    # has seq 2's own block 0 as parent, a different key: it is indexed
    assert a.stats()["cached_blocks"] == 3
    assert a.table(2) != a.table(1)
    # a new request follows the first chain
    assert a.add_cached(3, T) == 8 and a.table(3) == a.table(1)
    with pytest.raises(InvalidArg):
        a.add(9); a.append(9, 1); a.append_tokens(9, [1])   # no token history


# ---------------------------------------------------------------- swap
def test_swap_out_and_in_move_blocks_in_logical_order():
    bs = 4
    a = RefAllocator(8, bs, [7, 6, 5, 4, 3, 2, 1, 0])
    a.set_host_pool(4)
    a.add(1); a.append(1, 10)           # blocks 7, 6, 5
    a.add(2); a.append(2, 4)            # block 4
    pairs = a.swap_out(1)
    assert pairs == [(7, 0), (6, 1), (5, 2)]
    assert a.free_list() == [3, 2, 1, 0, 7, 6, 5]
    assert a.table(1) == [0, 1, 2] and a.length(1) == 10
    st = a.stats()
    assert st["host_free_blocks"] == 1 and st["swapped_seqs"] == 1 and st["used_blocks"] == 1
    with pytest.raises(InvalidArg):
        a.append(1, 1)
    with pytest.raises(InvalidArg):
        a.fork(1, 5)
    a.append(2, 8)                      # seq 2 now has 3 blocks, the host pool 1 free
    before = (list(a.free), list(a.host_free), a.table(2))
    with pytest.raises(OutOfBlocks):
        a.swap_out(2)
    assert before == (list(a.free), list(a.host_free), a.table(2))
    back = a.swap_in(1)                 # seq 2 took blocks 3, 2; the head is now 1, 0, 7
    assert back == [(0, 1), (1, 0), (2, 7)]
    assert a.table(1) == [1, 0, 7] and a.stats()["host_free_blocks"] == 4
    assert list(a.host_free) == [3, 0, 1, 2]


def test_swap_of_a_shared_block_keeps_the_other_owner():
    bs = 4
    a = RefAllocator(8, bs)
    a.set_host_pool(4)
    a.add(1); a.append(1, 6)
    a.fork(1, 2)
    pairs = a.swap_out(2)
    assert [d for d, _ in pairs] == a.table(1)
    assert all(a.ref[b] == 1 for b in a.table(1))
    a.free_seq(2)                       # a swapped sequence returns its host blocks
    assert a.stats()["host_free_blocks"] == 4 and a.stats()["swapped_seqs"] == 0
