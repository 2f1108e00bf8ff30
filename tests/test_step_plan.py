"""pa_step_plan -- one step's allocator events in one call, written into a
staging buffer -- against the oracle's allocator model (oracle/alloc_ref.py):
slots, copy-on-write pairs, table rows, lengths, free lists and refcounts
must be bit-exact, and the pair index per event must split the pairs where
the op-by-op calls would."""
import copy
import random

import numpy as np
import pytest

from oracle.alloc_ref import AllocError, RefAllocator, SeqTooLong
from paged_kv_cache_347_b200 import pagedattn as pa
from paged_kv_cache_347_b200.runner import PagedKVRunner
import workloads

EV = {"add": pa.EV_ADD, "free": pa.EV_FREE, "fork": pa.EV_FORK, "append": pa.EV_APPEND,
      "decode": pa.EV_DECODE}


def _encode(ops):
    ev, ids = [], np.empty(0, np.int64)
    for op in ops:
        if op[0] == "decode":
            ev.append((pa.EV_DECODE, 0, 0))
            ids = np.asarray(op[1], np.int64)
        elif op[0] in ("add", "free"):
            ev.append((EV[op[0]], op[1], 0))
        else:
            ev.append((EV[op[0]], op[1], op[2]))
    return np.asarray(ev, np.int64).reshape(-1, 3), ids


def _oracle_step(ref: RefAllocator, ops, width):
    """The documented semantics on the oracle: events in order, a run of
    consecutive appends all or nothing.  Returns (slots, pairs, pairs_before,
    tables, lens, applied, error code or 0)."""
    slots, pairs, pb = [], [], []
    tables = lens = None
    i = 0
    while i < len(ops):
        op = ops[i]
        if op[0] == "append":
            j = i
            while j < len(ops) and ops[j][0] == "append":
                j += 1
            snap = copy.deepcopy(ref.__dict__)
            run_slots, run_pairs, run_pb = [], [], []
            try:
                for k in range(i, j):
                    run_pb.append(len(pairs) + len(run_pairs))
                    s, p = ref.append(ops[k][1], ops[k][2])
                    run_slots += list(s)
                    if p:
                        run_pairs.append(tuple(p))
            except AllocError as e:
                ref.__dict__.clear()
                ref.__dict__.update(snap)
                return slots, pairs, pb, tables, lens, i, type(e).code
            slots += run_slots
            pairs += run_pairs
            pb += run_pb
            i = j
            continue
        pb.append(len(pairs))
        try:
            if op[0] == "add":
                ref.add(op[1])
            elif op[0] == "free":
                ref.free_seq(op[1])
            elif op[0] == "fork":
                ref.fork(op[1], op[2])
            else:
                rows = []
                for s in op[1]:
                    t = ref.table(s)
                    if len(t) > width:
                        raise SeqTooLong("table wider than width")
                    rows.append(t + [0] * (width - len(t)))
                tables = np.asarray(rows, np.int32).reshape(len(op[1]), width)
                lens = np.asarray([ref.length(s) for s in op[1]], np.int32)
        except AllocError as e:
            return slots, pairs, pb, tables, lens, i, type(e).code
        i += 1
    pb.append(len(pairs))
    return slots, pairs, pb, tables, lens, len(ops), 0


def _native_step(nat: pa.BlockAllocator, ops, width):
    ev, ids = _encode(ops)
    lay = nat.step_layout(ev, ids.size, width)
    stage = np.zeros(lay.bytes + 32, np.uint8)
    pb = np.full(ev.shape[0] + 1, -7, np.int32)
    code = 0
    try:
        lay = nat.step_plan(ev, ids, width, stage, pb)
    except pa.PagedAttnError as e:
        code = e.code
        lay = e.layout  # where the step stopped
    slots = stage[lay.off_slots:lay.off_slots + 8 * lay.n_slots].view(np.int64)
    pairs = stage[lay.off_pairs:lay.off_pairs + 16 * lay.n_pairs].view(np.int64).reshape(-1, 2)
    tables = stage[lay.off_tables:lay.off_tables + 4 * ids.size * width].view(np.int32)
    lens = stage[lay.off_lens:lay.off_lens + 4 * ids.size].view(np.int32)
    if code == 0 and ids.size:
        # the decode's dispatch order: rows longest first, ties in batch order
        order = stage[lay.off_order:lay.off_order + 4 * ids.size].view(np.int32)
        assert order.tolist() == np.argsort(-lens.astype(np.int64), kind="stable").tolist()
    return lay, slots, [tuple(int(x) for x in p) for p in pairs], pb, \
        tables.reshape(ids.size, width), lens, code


def _same_rows(tab, ref_tab, lens, bs):
    """Table rows agree on every entry a kernel reads (those below each
    sequence's block count); the rest is unspecified."""
    for r, L in enumerate(lens):
        n = -(-int(L) // bs)
        assert tab[r, :n].tolist() == ref_tab[r, :n].tolist(), r


def _same_state(ref: RefAllocator, nat: pa.BlockAllocator):
    assert nat.free_list() == ref.free_list()
    for b in range(ref.num_blocks):
        assert nat.refcount(b) == ref.ref[b]
    for sid in ref.tables:
        t, L = nat.seq_block_table(sid)
        assert t == ref.table(sid) and L == ref.length(sid)


@pytest.mark.parametrize("name", ["mix", "beam", "llama", "tiny"])
def test_workload_steps_bit_exact(name):
    wl = {"mix": lambda: workloads.mix(block_size=8, steps=5, batch=48, pool_slots=1 << 17),
          "beam": lambda: workloads.beam(steps=18, num_blocks=1024),
          "llama": lambda: workloads.llama(steps=4, batch=6, num_blocks=2048),
          "tiny": workloads.tiny}[name]()
    width = {"mix": 8192 // 8 + 8, "beam": 152, "llama": 300, "tiny": 4}[name]
    sh = wl.shape
    ref = RefAllocator(sh.num_blocks, sh.block_size, list(sh.free_order))
    nat = pa.BlockAllocator(sh.num_blocks, sh.block_size, sh.free_order)
    for i, st in enumerate(wl.steps):
        r_slots, r_pairs, r_pb, r_tab, r_lens, r_n, r_code = _oracle_step(ref, st.ops, width)
        lay, slots, pairs, pb, tab, lens, code = _native_step(nat, st.ops, width)
        assert code == r_code == 0, (i, code, r_code)
        assert slots.tolist() == r_slots, i
        assert pairs == r_pairs, i
        assert pb.tolist() == r_pb, i
        assert lay.events_applied == r_n == len(st.ops)
        if r_tab is not None:
            assert np.array_equal(lens, r_lens)
            _same_rows(tab, r_tab, r_lens, sh.block_size)
            assert lay.max_seq_len == int(r_lens.max())
            # the decode splits the step: rows and pairs before it
            k = [j for j, op in enumerate(st.ops) if op[0] == "decode"][0]
            assert lay.n_pairs_pre == r_pb[k]
            assert lay.n_slots_pre == sum(op[2] for op in st.ops[:k] if op[0] == "append")
        _same_state(ref, nat)
    if name == "beam":  # the copy-on-write step and the second private block
        assert ref.stats()["used_blocks"] == 4 * (128 + 4 * 2)


@pytest.mark.parametrize("seed", range(10))
def test_random_event_streams_with_failures(seed):
    """Small pools, forks, frees and appends that run out of blocks or hit
    the table bound: on a failing event the call stops, the failing run of
    appends is undone and everything before stays -- exactly as the oracle
    applying the same events with a snapshot per run."""
    rr = random.Random(seed)
    nb, bs = rr.choice([(12, 4), (24, 2), (40, 8)])
    order = [int(x) for x in np.random.default_rng(seed).permutation(nb)]
    mx = rr.choice([0, 6])
    ref = RefAllocator(nb, bs, order, mx)
    nat = pa.BlockAllocator(nb, bs, order, mx)
    live, nxt = [], 0
    width = 16
    for step in range(40):
        ops = []
        for _ in range(rr.randint(1, 6)):
            r = rr.random()
            if r < 0.25 or not live:
                ops.append(("add", nxt))
                live.append(nxt)
                nxt += 1
            elif r < 0.35:
                ops.append(("fork", rr.choice(live), nxt))
                live.append(nxt)
                nxt += 1
            elif r < 0.45:
                s = rr.choice(live)
                ops.append(("free", s))
                live.remove(s)
            else:
                ops.append(("append", rr.choice(live), rr.choice([0, 1, 1, 2, 5, 9])))
        if rr.random() < 0.6 and live:
            at = rr.randint(0, len(ops))
            ops.insert(at, ("decode", rr.sample(live, min(len(live), 3))))
            # a decode of a sequence freed or not yet added later in the step
            # is an error too; keep the decode batch valid at its position
            alive = set(x for x in range(nxt))
            for op in ops[:at]:
                if op[0] == "free":
                    alive.discard(op[1])
            added_after = {op[1] for op in ops[at + 1:] if op[0] == "add"} | \
                          {op[2] for op in ops[at + 1:] if op[0] == "fork"}
            ids = [s for s in ops[at][1] if s in alive and s not in added_after]
            ops[at] = ("decode", ids)
        r_slots, r_pairs, r_pb, r_tab, r_lens, r_n, r_code = _oracle_step(ref, ops, width)
        lay, slots, pairs, pb, tab, lens, code = _native_step(nat, ops, width)
        assert code == r_code, (step, ops, code, r_code)
        if code == 0:
            assert slots.tolist() == r_slots and pairs == r_pairs and pb.tolist() == r_pb
            if r_tab is not None:
                assert np.array_equal(lens, r_lens)
                _same_rows(tab, r_tab, r_lens, bs)
        else:
            assert lay.events_applied == r_n, (step, lay.events_applied, r_n)
            assert pb[:r_n].tolist() == r_pb[:r_n]
        _same_state(ref, nat)
        # sequences the step added but whose events were not applied, or that
        # a failed step left behind, follow the oracle's own record
        live = sorted(ref.tables.keys())


def test_bad_steps_are_refused_before_anything_is_applied():
    nat = pa.BlockAllocator(8, 4, None)
    nat.seq_add(1)
    before = (nat.free_list(), nat.seq_block_table(1))
    stage = np.zeros(4096, np.uint8)
    bad = [
        np.array([[pa.EV_APPEND, 1, 3], [9, 0, 0]], np.int64),                 # unknown code
        np.array([[pa.EV_DECODE, 0, 0], [pa.EV_DECODE, 0, 0]], np.int64),      # two decodes
        np.array([[pa.EV_APPEND, 1, -2]], np.int64),                           # negative count
    ]
    for ev in bad:
        with pytest.raises(pa.PagedAttnError) as e:
            nat.step_plan(ev, np.array([1], np.int64), 4, stage)
        assert e.value.code == -1
        assert (nat.free_list(), nat.seq_block_table(1)) == before
    # decode rows without a decode event
    with pytest.raises(pa.PagedAttnError):
        nat.step_plan(np.array([[pa.EV_APPEND, 1, 1]], np.int64), np.array([1], np.int64), 4,
                      stage)
    assert (nat.free_list(), nat.seq_block_table(1)) == before
    # a stage smaller than the layout
    ev = np.array([[pa.EV_APPEND, 1, 3], [pa.EV_DECODE, 0, 0]], np.int64)
    lay = nat.step_layout(ev, 1, 4)
    with pytest.raises(pa.PagedAttnError):
        nat.step_plan(ev, np.array([1], np.int64), 4, np.zeros(lay.bytes - 1, np.uint8))
    assert (nat.free_list(), nat.seq_block_table(1)) == before


def test_layout_depends_only_on_the_events_shape():
    """Offsets come from the events' kinds and counts (room for one pair per
    append event), never from what the allocator decides: the size query and
    the applied call agree, and every array starts 16-byte aligned."""
    nat = pa.BlockAllocator(64, 4, None)
    for s in range(3):
        nat.seq_add(s)
    ev = np.array([[pa.EV_APPEND, 0, 5], [pa.EV_APPEND, 1, 3], [pa.EV_FORK, 0, 7],
                   [pa.EV_APPEND, 7, 1], [pa.EV_DECODE, 0, 0], [pa.EV_APPEND, 2, 2]], np.int64)
    ids = np.array([0, 1, 7], np.int64)
    q = nat.step_layout(ev, 3, 10)
    stage = np.zeros(q.bytes, np.uint8)
    lay = nat.step_plan(ev, ids, 10, stage)
    for f in ("off_slots", "off_pairs", "off_tables", "off_lens", "bytes", "n_slots"):
        assert getattr(q, f) == getattr(lay, f), f
    for f in ("off_slots", "off_pairs", "off_tables", "off_lens"):
        assert getattr(lay, f) % 16 == 0
    assert lay.off_tables - lay.off_pairs >= 16 * 4   # four append events
    assert lay.n_slots == 11 and lay.n_slots_pre == 9
    # the fork shares sequence 0's partial last block: 7's append copies it
    assert lay.n_pairs == lay.n_pairs_pre == 1


def test_runner_splits_appends_at_every_other_event():
    """The runner's device actions keep the events' order: a fork between
    two appends ends a run, so the second run's copy reads the block after
    the first run's rows are written (as op-by-op planning does)."""
    r = PagedKVRunner.__new__(PagedKVRunner)
    enc = PagedKVRunner.encode_ops([("append", 0, 2), ("fork", 0, 5), ("append", 5, 1),
                                    ("append", 0, 1), ("decode", [0, 5]), ("free", 5),
                                    ("add", 9), ("append", 9, 4)])
    assert enc is not None
    assert enc.segments == [("write", 0, 1, 0, 2), ("write", 2, 4, 2, 4), ("decode", 4),
                            ("write", 7, 8, 4, 8)]
    assert PagedKVRunner.encode_ops([("admit", 3, [1, 2, 3])]) is None
    del r


def test_decode_order_is_longest_first_and_stable():
    assert pa.decode_order([5, 9, 9, 0, 14]).tolist() == [4, 1, 2, 0, 3]
    assert pa.decode_order([]).tolist() == []
    r = np.random.default_rng(0).integers(0, 50, size=300)
    assert pa.decode_order(r).tolist() == np.argsort(-r, kind="stable").tolist()
