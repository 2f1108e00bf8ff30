"""The C++ allocator behind the C ABI against the oracle allocator: slots,
copy-on-write pairs, tables, free lists and refcounts must be bit-exact."""
import random

import numpy as np
import pytest

from oracle.alloc_ref import AllocError, RefAllocator
from paged_kv_cache_347_b200 import pagedattn as pa
import workloads


def _same_state(ref: RefAllocator, nat: pa.BlockAllocator):
    assert nat.free_list() == ref.free_list()
    for b in range(ref.num_blocks):
        assert nat.refcount(b) == ref.ref[b]
    for sid in ref.tables:
        t, L = nat.seq_block_table(sid)
        assert t == ref.table(sid) and L == ref.length(sid)
    st = nat.stats()
    rs = ref.stats()
    for k, v in rs.items():
        assert st[k] == v, k


def _apply(ref, nat, op):
    """Applies op to both; returns (ref result or exception type, native ...)."""
    kind = op[0]
    r = n = None
    try:
        if kind == "add": ref.add(op[1])
        elif kind == "fork": ref.fork(op[1], op[2])
        elif kind == "free": ref.free_seq(op[1])
        elif kind == "append": r = ref.append(op[1], op[2])
    except AllocError as e:
        r = type(e).code
    try:
        if kind == "add": nat.seq_add(op[1])
        elif kind == "fork": nat.seq_fork(op[1], op[2])
        elif kind == "free": nat.seq_free(op[1])
        elif kind == "append":
            s, p = nat.seq_append(op[1], op[2])
            n = (s.tolist(), p)
    except pa.PagedAttnError as e:
        n = e.code
    if isinstance(r, tuple):
        r = (list(r[0]), r[1])
    assert r == n, (op, r, n)


@pytest.mark.parametrize("seed", range(8))
def test_random_ops_bit_exact(seed):
    rr = random.Random(seed)
    nb = rr.choice([8, 32, 64])
    bs = rr.choice([1, 2, 4, 8, 16, 32])
    order = list(np.random.default_rng(seed).permutation(nb))
    mx = rr.choice([0, 0, 5])
    ref = RefAllocator(nb, bs, order, mx)
    nat = pa.BlockAllocator(nb, bs, order, mx)
    live, nxt = [], 0
    for _ in range(600):
        x = rr.random()
        if x < 0.12 or not live:
            op = ("add", nxt); live.append(nxt); nxt += 1
        elif x < 0.65:
            op = ("append", rr.choice(live + [999]), rr.choice([0, 1, 1, 1, 2, 3, 9, 40]))
        elif x < 0.8:
            op = ("fork", rr.choice(live), rr.choice([nxt, live[0]]))
            if op[2] == nxt:
                live.append(nxt); nxt += 1
        else:
            s = rr.choice(live + [998]); op = ("free", s)
            if s in live:
                live.remove(s)
        _apply(ref, nat, op)
        _same_state(ref, nat)


def test_tiny_and_beam_event_lists_bit_exact():
    for wl in (workloads.tiny(), workloads.beam(steps=20)):
        sh = wl.shape
        ref = RefAllocator(sh.num_blocks, sh.block_size, sh.free_order)
        nat = pa.BlockAllocator(sh.num_blocks, sh.block_size, sh.free_order)
        for st in wl.steps:
            for op in st.ops:
                if op[0] != "decode":
                    _apply(ref, nat, op)
            _same_state(ref, nat)


def test_mix_event_list_batched_bit_exact():
    """Config-5-like churn at a reduced pool, through pa_batch_append."""
    wl = workloads.mix(block_size=8, steps=6, batch=32, pool_slots=8192 * 8)
    sh = wl.shape
    ref = RefAllocator(sh.num_blocks, sh.block_size, sh.free_order)
    nat = pa.BlockAllocator(sh.num_blocks, sh.block_size, sh.free_order)
    for st in wl.steps:
        ops = [op for op in st.ops if op[0] != "decode"]
        i = 0
        while i < len(ops):
            if ops[i][0] == "append":
                j = i
                while j < len(ops) and ops[j][0] == "append":
                    j += 1
                slots_ref, pairs_ref = [], []
                for op in ops[i:j]:
                    s, p = ref.append(op[1], op[2])
                    slots_ref += s
                    if p:
                        pairs_ref.append(p)
                s, p = nat.batch_append([o[1] for o in ops[i:j]], [o[2] for o in ops[i:j]])
                assert s.tolist() == slots_ref
                assert [tuple(x) for x in p.tolist()] == pairs_ref
                i = j
            else:
                _apply(ref, nat, ops[i])
                i += 1
        _same_state(ref, nat)


def test_batch_append_is_all_or_nothing():
    nat = pa.BlockAllocator(6, 4, list(range(6)))
    ref = RefAllocator(6, 4, list(range(6)))
    for a in (nat, ref):
        (a.seq_add if a is nat else a.add)(0)
    nat.seq_append(0, 6); ref.append(0, 6)            # blocks 0, 1
    nat.seq_fork(0, 1); ref.fork(0, 1)
    nat.seq_add(2); ref.add(2)
    before = (nat.free_list(), [nat.refcount(b) for b in range(6)])
    with pytest.raises(pa.PagedAttnError) as e:
        # seq 1 copies its shared block (1 block), seq 2 takes 2, seq 0 then 2 more: 5 > 4
        nat.batch_append([1, 2, 0], [1, 8, 8])
    assert e.value.code == -3
    assert (nat.free_list(), [nat.refcount(b) for b in range(6)]) == before
    _same_state(ref, nat)
    with pytest.raises(pa.PagedAttnError) as e:
        nat.batch_append([1, 77], [1, 1])
    assert e.value.code == -4
    _same_state(ref, nat)


def test_block_tables_export():
    nat = pa.BlockAllocator(16, 4, list(range(15, -1, -1)))
    for s, L in enumerate([5, 9, 14]):
        nat.seq_add(s); nat.seq_append(s, L)
    t, lens = nat.block_tables([2, 0], 4)
    assert lens.tolist() == [14, 5]
    assert t[0].tolist() == [10, 9, 8, 7] and t[1].tolist() == [15, 14, 0, 0]
    with pytest.raises(pa.PagedAttnError) as e:
        nat.block_tables([2], 3)
    assert e.value.code == -7


def test_create_validates_free_order():
    with pytest.raises(pa.PagedAttnError):
        pa.BlockAllocator(4, 4, [0, 1, 1, 2])
    with pytest.raises(pa.PagedAttnError):
        pa.BlockAllocator(0, 4)


def _apply_ext(ref, nat, op):
    """Prefix-cache and swap events on both allocators; results must agree."""
    kind = op[0]
    r = n = None
    try:
        if kind == "add_cached": r = ref.add_cached(op[1], op[2])
        elif kind == "admit":
            c = ref.add_cached(op[1], op[2])
            sl, p = ref.append_tokens(op[1], op[2][c:]); r = (c, list(sl), p)
        elif kind == "append_tokens":
            s, p = ref.append_tokens(op[1], op[2]); r = (list(s), p)
        elif kind == "swap_out": r = [tuple(x) for x in ref.swap_out(op[1])]
        elif kind == "swap_in": r = [tuple(x) for x in ref.swap_in(op[1])]
        else:
            return _apply(ref, nat, op)
    except AllocError as e:
        r = type(e).code
    try:
        if kind == "add_cached": n = nat.seq_add_cached(op[1], op[2])
        elif kind == "admit":
            c = nat.seq_add_cached(op[1], op[2])
            sl, p = nat.seq_append_tokens(op[1], op[2][c:]); n = (c, sl.tolist(), p)
        elif kind == "append_tokens":
            s, p = nat.seq_append_tokens(op[1], op[2]); n = (s.tolist(), p)
        elif kind == "swap_out": n = [tuple(x) for x in nat.seq_swap_out(op[1]).tolist()]
        elif kind == "swap_in": n = [tuple(x) for x in nat.seq_swap_in(op[1]).tolist()]
    except pa.PagedAttnError as e:
        n = e.code
    assert r == n, (op, r, n)


@pytest.mark.parametrize("seed", range(8))
def test_prefix_cache_and_swap_ops_bit_exact(seed):
    rr = random.Random(1000 + seed)
    nb = rr.choice([16, 32, 64])
    bs = rr.choice([1, 2, 4, 8])
    order = list(np.random.default_rng(seed).permutation(nb))
    ref = RefAllocator(nb, bs, order)
    nat = pa.BlockAllocator(nb, bs, order)
    hp = rr.choice([0, 8, 32])
    ref.set_host_pool(hp)
    nat.set_host_pool(hp)
    # a few shared "system prompts" so prefix hits happen
    prompts = [[rr.randrange(4) for _ in range(rr.randrange(bs, 5 * bs))] for _ in range(3)]
    live, nxt = [], 0
    for _ in range(500):
        x = rr.random()
        if x < 0.2 or not live:
            toks = rr.choice(prompts) + [rr.randrange(4) for _ in range(rr.randrange(0, 2 * bs))]
            op = (rr.choice(["admit", "admit", "add_cached"]), nxt, toks)
            live.append(nxt); nxt += 1
        elif x < 0.5:
            op = ("append_tokens", rr.choice(live), [rr.randrange(4) for _ in range(rr.choice([1, 1, 2, bs + 1]))])
        elif x < 0.6:
            op = ("append", rr.choice(live), rr.choice([1, 3]))
        elif x < 0.68:
            op = ("fork", rr.choice(live), nxt); live.append(nxt); nxt += 1
        elif x < 0.78:
            op = ("swap_out", rr.choice(live))
        elif x < 0.88:
            op = ("swap_in", rr.choice(live))
        else:
            s = rr.choice(live); op = ("free", s); live.remove(s)
        _apply_ext(ref, nat, op)
        _same_state(ref, nat)
    assert ref.stats()["prefix_hit_blocks"] > 0
