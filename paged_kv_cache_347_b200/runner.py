"""A decode-step driver over the C ABI: device caches plus the host allocator.

A step is a list of sequence events -- ("add", sid), ("fork", parent, child),
("free", sid), ("append", sid, n), ("decode", [sid, ...]) -- with the K/V
rows of its appends (in op order) and the queries of its decode.  The
runner turns a step into device actions in two phases:

* ``plan``: the C++ allocator runs every event on the host.  Consecutive
  appends (plain, with token ids, or the uncached part of an admitted
  sequence, whose cached rows get slot -1) become one ``write`` action: their
  slots and copy-on-write pairs.  A decode becomes a ``decode`` action
  carrying the block-table rows and lengths of its batch; a swap becomes a
  ``swap_out``/``swap_in`` action with its block pairs.  Any other event ends
  a run of appends, so the batched copies-then-writes of one action equal
  applying the appends one at a time.
* ``execute``: ``pa_copy_blocks`` (when the write has pairs), then
  ``pa_reshape_and_cache``, and for a decode ``pa_decode``; all on the
  current stream, nothing synchronised.

Each decode's kernel and split length: with ``partition_size`` -1 (the
default) and ``variant`` 0, pa_decode_choose's from the batch's lengths
(variant 3 with two KV heads per CTA on steps that read enough, else variant
2 with pa_decode_partition_for's split); a fixed ``partition_size`` (0 is
pa_decode's 512) or ``variant`` is kept as given.  The grid takes the batch
longest first, and a step's one-token appends go in with the decode
(pa_append_decode), unless ``longest_first`` / ``fuse_append`` are off.

``run`` does both for one step, moving the host arrays to the device on the
way.  Planning ahead lets a caller stage a whole run of steps in device
memory before timing it.
"""
from __future__ import annotations

import warnings
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

from . import pagedattn as pa


def _a256(x: int) -> int:
    return (x + 255) & ~255


@dataclass
class EncodedStep:
    """A step's events as pa_step_plan takes them: int64 [n, 3] triples
    {code, x, y} and the decode batch's sequence ids.  ``segments`` lists, in
    event order, each run of consecutive appends as ("write", first event,
    end event, first row, end row) and the decode as ("decode", index)."""
    events: np.ndarray
    decode_ids: np.ndarray
    segments: list = field(default_factory=list)

    def __post_init__(self):
        codes = self.events[:, 0]
        rows = np.concatenate([[0], np.cumsum(np.where(codes == pa.EV_APPEND,
                                                       self.events[:, 2], 0))])
        i, n = 0, codes.shape[0]
        while i < n:
            if codes[i] == pa.EV_APPEND:
                j = i
                while j < n and codes[j] == pa.EV_APPEND:
                    j += 1
                self.segments.append(("write", i, j, int(rows[i]), int(rows[j])))
                i = j
                continue
            if codes[i] == pa.EV_DECODE:
                self.segments.append(("decode", i))
            i += 1


@dataclass
class Action:
    kind: str                            # "write" | "decode" | "prefill" | "swap_out" | "swap_in"
    slots: Optional[np.ndarray] = None   # int64 [n]
    pairs: Optional[np.ndarray] = None   # int64 [k, 2]
    row0: int = 0
    nrows: int = 0
    tables: Optional[np.ndarray] = None  # int32 [b, width]
    lens: Optional[np.ndarray] = None    # int32 [b]
    max_len: int = 0
    cu: Optional[np.ndarray] = None      # prefill: int32 [b + 1] row offsets
    max_q: int = 0
    partition: int = 0                   # decode: split length passed to pa_decode
    variant: int = 0                     # decode: kernel (0 = pa_decode's own choice)
    hpc: int = 0                         # decode: KV heads per CTA (variant 3)
    order: Optional[np.ndarray] = None   # decode: int32 [b], rows longest first
    ids: Optional[np.ndarray] = None     # write of plain appends: their sequence ids
    ones: bool = False                   # write: every append was one token
    fused: bool = False                  # write: its rows go in with the next decode
    fuse: Optional["Action"] = None      # decode: the write fused into it
    dev: dict = field(default_factory=dict)


class PagedKVRunner:
    def __init__(self, num_blocks: int, block_size: int, num_heads: int, num_kv_heads: int,
                 head_dim: int, dtype: torch.dtype, scale: float, table_width: int,
                 free_order: Optional[Sequence[int]] = None, max_blocks_per_seq: int = 0,
                 device: str = "cuda", partition_size: int = -1, variant: int = 0,
                 prefill_variant: int = 0, longest_first: bool = True,
                 fuse_append: bool = True):
        self.alloc = pa.BlockAllocator(num_blocks, block_size, free_order, max_blocks_per_seq)
        self.device = torch.device(device)
        dims = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_cache = torch.zeros(dims, dtype=dtype, device=self.device)
        self.v_cache = torch.zeros(dims, dtype=dtype, device=self.device)
        self.num_heads, self.num_kv_heads, self.head_dim = num_heads, num_kv_heads, head_dim
        self.block_size, self.num_blocks = block_size, num_blocks
        self.dtype, self.scale, self.width = dtype, scale, table_width
        self.partition_size, self.variant = partition_size, variant
        self.prefill_variant = prefill_variant
        # decode grids take the batch's sequences longest first (seq_order)
        self.longest_first = longest_first
        # a decode step's one-token appends go in with the decode
        # (pa_append_decode) instead of a separate pa_reshape_and_cache
        self.fuse_append = fuse_append
        # host-fed steps: two staging slots (page-locked host / device buffer
        # pairs), the event after which each slot's host buffer is free, the
        # event after which each slot's device buffer is free, and the graphs
        # of the layouts seen so far with their two copy streams
        self._stage = [None, None]
        self._stage_ev = [None, None]
        self._run_ev = [None, None]
        self._next_slot = 0
        self._graphs = {}
        self._s_in = self._s_out = None

    @classmethod
    def for_shape(cls, shape, table_width: int, **kw) -> "PagedKVRunner":
        dt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[shape.dtype]
        return cls(shape.num_blocks, shape.block_size, shape.num_heads, shape.num_kv_heads,
                   shape.head_dim, dt, shape.scale, table_width, shape.free_order, **kw)

    # ------------------------------------------------------------ plan
    def enable_swap(self, num_host_blocks: int) -> None:
        """Host pool for swapped-out sequences: the allocator's host blocks and
        page-locked host caches of the same block shape."""
        self.alloc.set_host_pool(num_host_blocks)
        dims = (max(num_host_blocks, 1), self.num_kv_heads, self.block_size, self.head_dim)
        self.k_host = torch.zeros(dims, dtype=self.dtype).pin_memory()
        self.v_host = torch.zeros(dims, dtype=self.dtype).pin_memory()

    def plan(self, ops) -> List[Action]:
        acts: List[Action] = []
        row = 0
        pend = {"slots": [], "pairs": [], "row0": 0, "nrows": 0, "ids": None, "ones": False}

        def add_rows(slots, pairs, n):
            if pend["nrows"] == 0:
                pend["row0"] = row
            pend["slots"].append(np.asarray(slots, dtype=np.int64))
            if pairs is not None and len(pairs):
                pend["pairs"].append(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
            pend["nrows"] += n

        def flush():
            if pend["nrows"]:
                pairs = (np.concatenate(pend["pairs"]) if pend["pairs"]
                         else np.empty((0, 2), np.int64))
                acts.append(Action("write", slots=np.concatenate(pend["slots"]), pairs=pairs,
                                   row0=pend["row0"], nrows=pend["nrows"], ids=pend["ids"],
                                   ones=pend["ones"]))
            pend.update(slots=[], pairs=[], nrows=0, ids=None, ones=False)

        i = 0
        while i < len(ops):
            op = ops[i]
            kind = op[0]
            if kind == "append":
                ids, ns = [], []
                while i < len(ops) and ops[i][0] == "append":
                    ids.append(ops[i][1])
                    ns.append(ops[i][2])
                    i += 1
                slots, pairs = self.alloc.batch_append(ids, ns)
                n = int(sum(ns))
                plain = pend["nrows"] == 0
                add_rows(slots.copy(), pairs.copy(), n)
                if plain:  # a write of plain appends only (so far)
                    pend["ids"] = np.asarray(ids, np.int64)
                    pend["ones"] = all(x == 1 for x in ns)
                else:
                    pend["ids"] = None
                row += n
                continue
            if kind == "append_tokens":
                pend["ids"] = None
                slots, pair = self.alloc.seq_append_tokens(op[1], op[2])
                add_rows(slots.copy(), [pair] if pair else None, len(op[2]))
                row += len(op[2])
            elif kind == "admit":
                pend["ids"] = None
                toks = op[2]
                c = self.alloc.seq_add_cached(op[1], toks)
                slots, pair = self.alloc.seq_append_tokens(op[1], toks[c:])
                # rows of cached tokens are skipped (slot -1)
                add_rows(np.concatenate([np.full(c, -1, np.int64), slots]),
                         [pair] if pair else None, len(toks))
                row += len(toks)
            else:
                flush()
                if kind == "add":
                    self.alloc.seq_add(op[1])
                elif kind == "fork":
                    self.alloc.seq_fork(op[1], op[2])
                elif kind == "free":
                    self.alloc.seq_free(op[1])
                elif kind == "decode":
                    dec_ids = np.asarray(op[1], np.int64)
                    tables, lens = self.alloc.block_tables(list(op[1]), self.width)
                    part, var, hpc = self._choose(lens)
                    acts.append(Action("decode", tables=tables, lens=lens,
                                       max_len=int(lens.max()) if lens.size else 0,
                                       partition=part, variant=var, hpc=hpc,
                                       order=pa.decode_order(lens) if self.longest_first
                                       else None, ids=dec_ids))
                elif kind == "prefill":
                    sids = [x for x, _ in op[1]]
                    ns = np.array([n for _, n in op[1]], np.int32)
                    tables, lens = self.alloc.block_tables(sids, self.width)
                    a = Action("prefill", tables=tables, lens=lens,
                               max_len=int(lens.max()) if lens.size else 0)
                    a.cu = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
                    a.max_q = int(ns.max()) if ns.size else 0
                    acts.append(a)
                elif kind == "host_pool":
                    self.enable_swap(op[1])
                elif kind == "swap_out":
                    acts.append(Action("swap_out", pairs=self.alloc.seq_swap_out(op[1])))
                elif kind == "swap_in":
                    acts.append(Action("swap_in", pairs=self.alloc.seq_swap_in(op[1])))
                else:
                    raise ValueError(f"unknown op {op!r}")
            i += 1
        flush()
        self._mark_fusable(acts)
        return acts

    def _mark_fusable(self, acts: List[Action]) -> None:
        """A write of one-token appends of exactly the decode batch, in its
        order, right before the decode, goes in with it (pa_append_decode)."""
        if not self.fuse_append:
            return
        for i in range(1, len(acts)):
            w, d = acts[i - 1], acts[i]
            if (d.kind == "decode" and w.kind == "write" and w.ones and w.ids is not None
                    and w.nrows == d.tables.shape[0] and d.ids is not None
                    and np.array_equal(w.ids, d.ids)):
                w.fused, d.fuse = True, w

    # ------------------------------------------------------------ device side
    def upload(self, acts: List[Action], pin: bool = False) -> None:
        """Copy each action's host arrays to the device (async from pinned
        memory when ``pin``)."""
        def put(a: np.ndarray) -> torch.Tensor:
            t = torch.from_numpy(np.ascontiguousarray(a))
            if pin:
                t = t.pin_memory()
            return t.to(self.device, non_blocking=pin)

        for a in acts:
            if a.kind == "write":
                a.dev["slots"] = put(a.slots)
                if len(a.pairs):
                    a.dev["pairs"] = put(a.pairs)
            elif a.kind in ("decode", "prefill"):
                a.dev["tables"] = put(a.tables)
                a.dev["lens"] = put(a.lens)
                if a.kind == "prefill":
                    a.dev["cu"] = put(a.cu)
                elif a.order is not None:
                    a.dev["order"] = put(a.order)
            elif len(a.pairs):
                a.dev["pairs"] = put(a.pairs)

    def execute(self, acts: List[Action], k_new: Optional[torch.Tensor],
                v_new: Optional[torch.Tensor], q: Optional[torch.Tensor],
                out: Optional[torch.Tensor] = None) -> Optional[torch.Tensor]:
        res = None
        for a in acts:
            if a.kind == "write":
                if "pairs" in a.dev:
                    pa.pa_copy_blocks(self.k_cache, self.v_cache, a.dev["pairs"])
                if a.nrows and not a.fused:
                    pa.pa_reshape_and_cache(k_new[a.row0:a.row0 + a.nrows],
                                            v_new[a.row0:a.row0 + a.nrows], self.k_cache,
                                            self.v_cache, a.dev["slots"])
            elif a.kind == "prefill":
                o = torch.empty((int(a.cu[-1]), self.num_heads, self.head_dim),
                                dtype=torch.float32, device=self.device)
                pa.pa_prefill(o, q, self.k_cache, self.v_cache, a.dev["tables"], a.dev["lens"],
                              a.dev["cu"], self.scale, max_q_len=a.max_q,
                              max_seq_len=a.max_len, variant=self.prefill_variant)
                res = o
            elif a.kind == "swap_out":
                if "pairs" in a.dev:
                    pa.pa_swap_blocks(self.k_host, self.v_host, self.k_cache, self.v_cache,
                                      a.dev["pairs"])
            elif a.kind == "swap_in":
                if "pairs" in a.dev:
                    pa.pa_swap_blocks(self.k_cache, self.v_cache, self.k_host, self.v_host,
                                      a.dev["pairs"])
            else:
                b = a.tables.shape[0]
                o = out if out is not None else torch.empty(
                    (b, self.num_heads, self.head_dim), dtype=torch.float32, device=self.device)
                if a.fuse is not None:
                    w = a.fuse
                    pa.pa_append_decode(o, q, k_new[w.row0:w.row0 + b], v_new[w.row0:w.row0 + b],
                                        w.dev["slots"], self.k_cache, self.v_cache,
                                        a.dev["tables"], a.dev["lens"], self.scale,
                                        max_seq_len=a.max_len, partition_size=a.partition,
                                        variant=a.variant, heads_per_cta=a.hpc,
                                        seq_order=a.dev.get("order"))
                else:
                    pa.pa_decode(o, q, self.k_cache, self.v_cache, a.dev["tables"],
                                 a.dev["lens"], self.scale, max_seq_len=a.max_len,
                                 partition_size=a.partition, variant=a.variant,
                                 heads_per_cta=a.hpc, seq_order=a.dev.get("order"))
                res = o
        return res

    # ------------------------------------------------------------ host-fed steps
    # A step fed from host memory is split in two so that the host work of the
    # next step (allocator, table rows) can run while the GPU works on this one:
    #   prepare(ops)  -> host only: pa_step_plan applies the step's events and
    #                    writes slots, copy pairs, table rows and lengths
    #                    straight into one of two page-locked staging buffers
    #                    (steps with ops it does not take -- prefix-cached
    #                    admissions, swaps, prefills -- are planned op by op
    #                    and packed into the same buffer);
    #   launch(...)   -> one copy of the staging buffer, one copy each of the
    #                    new K/V rows and queries, the kernels, the output
    #                    copied back into page-locked memory -- all asynchronous;
    #   wait()        -> synchronise (the output is then readable).
    @staticmethod
    def encode_ops(ops) -> Optional[EncodedStep]:
        """The step's events as pa_step_plan takes them, or None when the
        step has an op that it does not take."""
        if isinstance(ops, EncodedStep):
            return ops
        ev, ids = [], None
        for op in ops:
            k = op[0]
            if k == "append":
                ev.append((pa.EV_APPEND, op[1], op[2]))
            elif k == "add":
                ev.append((pa.EV_ADD, op[1], 0))
            elif k == "free":
                ev.append((pa.EV_FREE, op[1], 0))
            elif k == "fork":
                ev.append((pa.EV_FORK, op[1], op[2]))
            elif k == "decode" and ids is None:
                ev.append((pa.EV_DECODE, 0, 0))
                ids = np.asarray(op[1], dtype=np.int64)
            else:
                return None
        return EncodedStep(np.asarray(ev, dtype=np.int64).reshape(-1, 3),
                           np.empty(0, np.int64) if ids is None else ids)

    def _staging(self, slot: int, nbytes: int):
        """Pinned host / device buffer pair number ``slot`` (of 2), grown on demand."""
        cur = self._stage[slot]
        if cur is None or cur[0].numel() < nbytes:
            n = max(nbytes, 1 << 20)
            if self._stage_ev[slot] is not None:
                self._stage_ev[slot].synchronize()
            if self._run_ev[slot] is not None:
                self._run_ev[slot].synchronize()
            cur = (torch.empty(n, dtype=torch.uint8).pin_memory(),
                   torch.empty(n, dtype=torch.uint8, device=self.device))
            self._stage[slot] = cur
            self._stage_ev[slot] = None
        if self._stage_ev[slot] is not None:
            self._stage_ev[slot].synchronize()  # its previous copy has left the host buffer
        return cur

    def _input_bytes(self, n_rows: int, b: int) -> int:
        e = torch.tensor([], dtype=self.dtype).element_size()
        kv = n_rows * self.num_kv_heads * self.head_dim * e
        return 2 * _a256(kv) + _a256(b * self.num_heads * self.head_dim * e)

    def prepare(self, ops) -> dict:
        """Host half of a step: the allocator's work and every array the
        step's kernels read, in a page-locked staging buffer."""
        enc = self.encode_ops(ops)
        if enc is None:
            return self._prepare_ops(ops)
        b = int(enc.decode_ids.size)
        slot = self._next_slot
        self._next_slot = 1 - slot
        host, devb = self._staging(slot, 0)
        hb = host.numpy()
        pb = np.empty(enc.events.shape[0] + 1, np.int32)
        try:
            lay = self.alloc.step_plan(enc.events, enc.decode_ids, self.width, hb, pb)
        except pa.PagedAttnError as e:
            need = e.layout.bytes if e.code == -1 else 0
            if need <= hb.nbytes:
                raise
            # too small a buffer is refused before anything is applied: grow,
            # with room behind the arrays for the step's new rows and queries
            host, devb = self._staging(slot, _a256(need) + self._input_bytes(e.layout.n_slots, b))
            hb = host.numpy()
            lay = self.alloc.step_plan(enc.events, enc.decode_ids, self.width, hb, pb)
        slots = hb[lay.off_slots:lay.off_slots + 8 * lay.n_slots].view(np.int64)
        pairs = hb[lay.off_pairs:lay.off_pairs + 16 * lay.n_pairs].view(np.int64).reshape(-1, 2)
        acts, arrays, offs = [], [], []
        # device actions in event order: each run of appends is its copies,
        # then its rows (as op-by-op planning makes them); the decode in place
        for seg in enc.segments:
            if seg[0] == "write":
                _, e0, e1, r0, r1 = seg
                p0, p1 = int(pb[e0]), int(pb[e1])
                ev = enc.events[e0:e1]
                w = Action("write", slots=slots[r0:r1], pairs=pairs[p0:p1], row0=r0,
                           nrows=r1 - r0, ids=ev[:, 1], ones=bool((ev[:, 2] == 1).all()))
                acts.append(w)
                if r1 > r0:
                    arrays.append((w, "slots", w.slots))
                    offs.append(lay.off_slots + 8 * r0)
                if p1 > p0:
                    arrays.append((w, "pairs", w.pairs))
                    offs.append(lay.off_pairs + 16 * p0)
            else:
                tables = hb[lay.off_tables:lay.off_tables + 4 * b * self.width].view(np.int32)
                tables = tables.reshape(b, self.width)
                lens = hb[lay.off_lens:lay.off_lens + 4 * b].view(np.int32)
                order = hb[lay.off_order:lay.off_order + 4 * b].view(np.int32)
                part, var, hpc = self._choose(lens)
                d = Action("decode", tables=tables, lens=lens.copy(), max_len=lay.max_seq_len,
                           partition=part, variant=var, hpc=hpc,
                           order=order if self.longest_first else None, ids=enc.decode_ids)
                acts.append(d)
                arrays += [(d, "tables", tables), (d, "lens", lens)]
                offs += [lay.off_tables, lay.off_lens]
                if self.longest_first:
                    arrays.append((d, "order", order))
                    offs.append(lay.off_order)
        self._mark_fusable(acts)
        return {"acts": acts, "arrays": arrays, "offs": offs, "bytes": lay.bytes, "slot": slot,
                "host": host, "dev": devb}

    def _choose(self, lens: np.ndarray):
        """(split length, kernel, KV heads per CTA) of a decode: the runner's
        fixed choices, else the library's for these lengths
        (pa_decode_choose / pa_decode_partition_for)."""
        part, var = self.partition_size, self.variant
        if part >= 0:
            return part, var, 0
        if var == 0:
            return pa.decode_choose(lens, self.num_kv_heads, self.head_dim, self.block_size,
                                    self.dtype)
        part = pa.decode_partition_for(lens, self.num_kv_heads, self.head_dim,
                                       self.block_size, self.dtype)
        return part, var, 0

    def _prepare_ops(self, ops) -> dict:
        """prepare() for steps pa_step_plan does not take: plan op by op,
        then pack the arrays into the staging buffer."""
        acts = self.plan(ops)
        arrays = []
        for a in acts:
            if a.kind == "write":
                arrays.append((a, "slots", a.slots))
                if len(a.pairs):
                    arrays.append((a, "pairs", a.pairs))
            elif a.kind in ("decode", "prefill"):
                arrays.append((a, "tables", a.tables))
                arrays.append((a, "lens", a.lens))
                if a.kind == "prefill":
                    arrays.append((a, "cu", a.cu))
                elif a.order is not None:
                    arrays.append((a, "order", a.order))
            elif len(a.pairs):
                arrays.append((a, "pairs", a.pairs))
        offs, total = [], 0
        for _, _, arr in arrays:
            offs.append(total)
            total += (arr.nbytes + 15) & ~15
        slot = self._next_slot
        self._next_slot = 1 - slot
        host, devb = self._staging(slot, total)
        hb = host.numpy()
        for (_, _, arr), off in zip(arrays, offs):
            hb[off:off + arr.nbytes] = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
        return {"acts": acts, "arrays": arrays, "offs": offs, "bytes": total, "slot": slot,
                "host": host, "dev": devb}

    def _bind(self, prep: dict) -> None:
        """Point each action's device arrays into the slot's device buffer."""
        devb = prep["dev"]
        for (a, name, arr), off in zip(prep["arrays"], prep["offs"]):
            dt = torch.int64 if arr.dtype == np.int64 else torch.int32
            a.dev[name] = devb[off:off + arr.nbytes].view(dt).view(arr.shape)

    def launch(self, prep: dict, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
               out_host: torch.Tensor) -> dict:
        """Device half of a step, all asynchronous on the current stream."""
        total, host, devb = prep["bytes"], prep["host"], prep["dev"]
        if total:
            devb[:total].copy_(host[:total], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record()
            self._stage_ev[prep["slot"]] = ev
        self._bind(prep)
        dev = [t.to(self.device, non_blocking=True) for t in (k_new, v_new, q)]
        o = self.execute(prep["acts"], *dev)
        ev_run = torch.cuda.Event()
        ev_run.record()
        self._run_ev[prep["slot"]] = ev_run  # a graph step's copy in waits for it
        out_host.copy_(o, non_blocking=True)
        h2d = total + sum(t.nbytes for t in (k_new, v_new, q))
        return {"h2d": h2d, "d2h": out_host.nbytes, "acts": prep["acts"]}

    def wait(self) -> None:
        """Synchronise the current stream and the graph steps' copy streams."""
        torch.cuda.current_stream(self.device).synchronize()
        if self._s_out is not None:
            self._s_in.synchronize()
            self._s_out.synchronize()

    # ------------------------------------------------------------ graph replay
    # Steps of the same layout (the same action kinds and sizes, no copy-on-
    # write pairs, prepared in the same staging slot) repeat the same device
    # work on different bytes.  The kernels of a layout are captured once, as
    # a graph, and the output's copy back as another; a replay copies the
    # slot's staging buffer and the step's new K/V rows and queries to fixed
    # places in the slot's device buffer on a copy stream, runs the kernels'
    # graph on the current stream and the copy back on a second copy stream.
    # A decode inside a graph takes a length bound of the step's longest
    # sequence rounded up to a power of two (at least 512 tokens, at most the
    # table's capacity), so that its grid is fixed while steps change little.
    @staticmethod
    def _graphable(acts) -> bool:
        return (bool(acts) and all(a.kind in ("write", "decode") for a in acts)
                and not any(a.kind == "write" and len(a.pairs) for a in acts)
                and sum(a.kind == "decode" for a in acts) == 1)

    def _graph_bound(self, max_len: int) -> int:
        cap = self.width * self.block_size
        bound = 512
        while bound < max_len:
            bound *= 2
        return min(bound, cap)

    def _graph_key(self, prep: dict, k_new: torch.Tensor, q: torch.Tensor):
        acts = prep["acts"]
        layout = tuple((a.kind, a.nrows, None if a.tables is None else a.tables.shape,
                        a.partition, a.variant, a.hpc,
                        self._graph_bound(a.max_len) if a.kind == "decode" else 0,
                        a.order is not None, a.fused, a.fuse is not None)
                       for a in acts)
        return (layout, prep["bytes"], prep["slot"], prep["dev"].data_ptr(),
                tuple(k_new.shape), tuple(q.shape), k_new.dtype)

    def _input_offsets(self, prep: dict, k_new: torch.Tensor, v_new: torch.Tensor,
                       q: torch.Tensor):
        """Fixed places for the step's new K/V rows and queries in the slot's
        device buffer, behind its arrays (256-byte aligned); the buffers grow,
        keeping the arrays, when too small."""
        total = prep["bytes"]
        offs, end = [], _a256(total)
        for t in (k_new, v_new, q):
            offs.append(end)
            end = _a256(end + t.nbytes)
        if prep["dev"].numel() < end:
            old = prep["host"]
            prep["host"], prep["dev"] = self._staging(prep["slot"], end)
            prep["host"][:total].copy_(old[:total])
        return offs

    def _capture(self, prep: dict, k_new: torch.Tensor, v_new: torch.Tensor,
                 q: torch.Tensor, offs) -> dict:
        dec = [a for a in prep["acts"] if a.kind == "decode"][0]
        devb, host, total = prep["dev"], prep["host"], prep["bytes"]
        ins = [devb[off:off + t.nbytes].view(t.dtype).view(t.shape)
               for off, t in zip(offs, (k_new, v_new, q))]
        g = {"out": torch.empty((dec.tables.shape[0], self.num_heads, self.head_dim),
                                dtype=torch.float32).pin_memory(),
             "in_bytes": sum(t.nbytes for t in (k_new, v_new, q)), "ins": ins}
        for a in prep["acts"]:
            if a.kind == "decode":
                a.max_len = self._graph_bound(a.max_len)

        def body_run():
            self._bind(prep)
            g["o"] = self.execute(prep["acts"], *ins)

        def body_out():
            g["out"].copy_(g["o"], non_blocking=True)

        # one eager run first (workspace, per-device set-up); it applies this
        # step, and the replay applies it again to the same bytes
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            if total:
                devb[:total].copy_(host[:total], non_blocking=True)
            for dst, src in zip(ins, (k_new, v_new, q)):
                dst.copy_(src, non_blocking=True)
            body_run()
            body_out()
        side.synchronize()
        # the graph writes split partials into the binding's cached workspace:
        # keep that buffer alive for as long as the graph
        g["ws"] = pa.cached_workspace(self.device)
        for name, body in (("g_run", body_run), ("g_out", body_out)):
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=side, capture_error_mode="thread_local"):
                body()
            g[name] = graph
        g["exec_run"] = g["g_run"].raw_cuda_graph_exec()
        g["exec_out"] = g["g_out"].raw_cuda_graph_exec()
        # events re-recorded at every replay of this layout (made, and recorded
        # once so that they exist, here: the host side of a replay stays short)
        g["ev_in"], g["ev_run"], g["ev_out"] = (torch.cuda.Event() for _ in range(3))
        with torch.cuda.stream(side):
            for ev in (g["ev_in"], g["ev_run"], g["ev_out"]):
                ev.record()
        side.synchronize()
        # the copies in: the staging buffer's arrays, then the new rows and
        # queries (their sources are set per step)
        c = (pa.pa_host_copy * 4)()
        c[0].dst, c[0].src, c[0].bytes = devb.data_ptr(), host.data_ptr(), total
        for i, (off, t) in enumerate(zip(offs, (k_new, v_new, q)), start=1):
            c[i].dst, c[i].bytes = devb.data_ptr() + off, t.nbytes
        g["copies"] = c
        g["replayed"] = False
        return g

    def stage_graph(self, prep: dict, k_new: torch.Tensor, v_new: torch.Tensor,
                    q: torch.Tensor) -> Optional[dict]:
        """Graph of this step's layout, captured the first time (which runs
        the step once eagerly); None when the layout has no graph form.  The
        step's inputs are remembered for replay_graph, which copies them: they
        must stay unchanged until the step's "ready" event."""
        if not self._graphable(prep["acts"]):
            return None
        offs = self._input_offsets(prep, k_new, v_new, q)
        key = self._graph_key(prep, k_new, q)
        if key in self._graphs and self._graphs[key] is None:
            return None  # this layout failed to capture before: launch eagerly
        g = self._graphs.get(key)
        if g is None:
            try:
                g = self._capture(prep, k_new, v_new, q, offs)
            except RuntimeError as e:  # capture refused: this layout runs eagerly
                warnings.warn(f"CUDA graph capture failed, launching eagerly: {e}")
                self._graphs[key] = None
                torch.cuda.synchronize(self.device)
                return None
            self._graphs[key] = g
            prep["captured"] = True
        prep["inputs"] = (k_new, v_new, q)
        return g

    def _copy_streams(self):
        if self._s_in is None:
            self._s_in = torch.cuda.Stream(self.device)
            self._s_out = torch.cuda.Stream(self.device)
            self._s_handles = (self._s_in.cuda_stream, self._s_out.cuda_stream)
        return self._s_in, self._s_out

    def replay_graph(self, g: dict, prep: dict) -> dict:
        """Device half of a graph step, one library call (pa_step_launch): the
        copies in run on a copy stream once the previous step of this staging
        slot has finished with the slot's device buffer; the kernels' graph
        runs on the current stream after them (and after this layout's
        previous output has been copied out); the output's copy graph runs on
        a second copy stream.  The output lands in a page-locked tensor owned
        by the graph, readable once the returned "ready" event has completed
        (or after wait()) until the next replay of the same layout."""
        self._copy_streams()
        c = g["copies"]
        k, v, q = prep["inputs"]
        c[1].src, c[2].src, c[3].src = k.data_ptr(), v.data_ptr(), q.data_ptr()
        slot = prep["slot"]
        prev = self._run_ev[slot]
        pa.step_launch(self._s_handles[0], torch.cuda.current_stream(self.device).cuda_stream,
                       self._s_handles[1], c, 4, prev.cuda_event if prev is not None else 0,
                       g["ev_in"].cuda_event, g["exec_run"],
                       g["ev_out"].cuda_event if g["replayed"] else 0, g["ev_run"].cuda_event,
                       g["exec_out"], g["ev_out"].cuda_event)
        self._stage_ev[slot] = g["ev_in"]  # the host staging buffer is free again after this
        self._run_ev[slot] = g["ev_run"]
        g["replayed"] = True
        return {"h2d": prep["bytes"] + g["in_bytes"], "d2h": g["out"].nbytes,
                "acts": prep["acts"], "out": g["out"], "ready": g["ev_out"]}

    def launch_graph(self, prep: dict, k_new: torch.Tensor, v_new: torch.Tensor,
                     q: torch.Tensor) -> Optional[dict]:
        """stage_graph + replay_graph; None (nothing launched) when the step's
        layout has no graph form."""
        g = self.stage_graph(prep, k_new, v_new, q)
        return None if g is None else self.replay_graph(g, prep)

    def run_pinned(self, ops, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                   out_host: torch.Tensor) -> dict:
        """prepare + launch + wait for one step fed from pinned host memory."""
        res = self.launch(self.prepare(ops), k_new, v_new, q, out_host)
        self.wait()
        return res

    def run(self, step) -> Optional[torch.Tensor]:
        """Plan, upload and execute one step whose tensors may live on the host."""
        acts = self.plan(step.ops)
        self.upload(acts)
        to = lambda t: None if t is None else t.to(self.device)
        return self.execute(acts, to(step.k_new), to(step.v_new), to(step.q))
