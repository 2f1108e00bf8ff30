"""Walk a ``workloads`` event list through the oracle -- TEST INFRASTRUCTURE ONLY.

Each ``append`` op asks the reference allocator for its slots (and a
copy-on-write pair, applied to the host caches before the new rows are
written), then scatters that op's K/V rows; each ``decode`` op evaluates the
fp64 paged attention of the step's queries over the current caches.  Ops run
one at a time in list order.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

from workloads import DTYPES, Shape, Step

from . import attn, cache_ref
from .alloc_ref import RefAllocator


class OracleRun:
    def __init__(self, shape: Shape, max_blocks_per_seq: int = 0, keep_cache: bool = True):
        self.shape = shape
        self.alloc = RefAllocator(shape.num_blocks, shape.block_size, shape.free_order,
                                  max_blocks_per_seq)
        dims = (shape.num_blocks, shape.num_kv_heads, shape.block_size, shape.head_dim)
        dt = DTYPES[shape.dtype]
        self.keep_cache = keep_cache
        self.k_cache = torch.zeros(dims, dtype=dt) if keep_cache else None
        self.v_cache = torch.zeros(dims, dtype=dt) if keep_cache else None

    def tables(self, sids: Sequence[int], width: int = 0) -> Tuple[np.ndarray, np.ndarray]:
        rows = [self.alloc.table(s) for s in sids]
        w = max([width] + [len(r) for r in rows] + [1])
        bt = np.zeros((len(sids), w), np.int32)
        for i, r in enumerate(rows):
            bt[i, :len(r)] = r
        lens = np.array([self.alloc.length(s) for s in sids], np.int32)
        return bt, lens

    def step(self, st: Step, sel: Optional[Sequence[Tuple[int, int]]] = None,
             decode: bool = True, n_threads: int = 0) -> Dict:
        """Apply one step.  Returns the slots and copy-on-write pairs of its
        appends (in op order) and, when ``decode``, the fp64 outputs of its
        decode op ([b, Hq, D], or [len(sel), D] for (batch index, head) pairs)
        or of its prefill op ([rows, Hq, D], or [len(sel), D] for (row, head)
        pairs)."""
        res: Dict = {"slots": [], "pairs": [], "out": None}
        row = 0
        for op in st.ops:
            kind = op[0]
            if kind == "add":
                self.alloc.add(op[1])
            elif kind == "fork":
                self.alloc.fork(op[1], op[2])
            elif kind == "free":
                self.alloc.free_seq(op[1])
            elif kind in ("append", "append_tokens", "admit"):
                sid = op[1]
                if kind == "append":
                    n = op[2]
                    slots, pair = self.alloc.append(sid, n)
                elif kind == "append_tokens":
                    n = len(op[2])
                    slots, pair = self.alloc.append_tokens(sid, op[2])
                else:
                    n = len(op[2])
                    c = self.alloc.add_cached(sid, op[2])
                    slots, pair = self.alloc.append_tokens(sid, op[2][c:])
                    slots = [-1] * c + list(slots)   # cached rows are not written
                res["slots"] += slots
                if pair is not None:
                    res["pairs"].append(pair)
                if self.keep_cache:
                    if pair is not None:
                        cache_ref.copy_blocks(self.k_cache, self.v_cache, [pair])
                    cache_ref.reshape_and_cache(st.k_new[row:row + n], st.v_new[row:row + n],
                                                self.k_cache, self.v_cache, slots)
                row += n
            elif kind == "host_pool":
                self.alloc.set_host_pool(op[1])
                if self.keep_cache:
                    dims = (max(op[1], 1),) + tuple(self.k_cache.shape[1:])
                    self.k_host = torch.zeros(dims, dtype=self.k_cache.dtype)
                    self.v_host = torch.zeros(dims, dtype=self.k_cache.dtype)
            elif kind == "swap_out":
                pairs = self.alloc.swap_out(op[1])
                res.setdefault("swaps", []).append(("out", pairs))
                if self.keep_cache:
                    cache_ref.copy_between(self.k_host, self.v_host, self.k_cache, self.v_cache,
                                           pairs)
            elif kind == "swap_in":
                pairs = self.alloc.swap_in(op[1])
                res.setdefault("swaps", []).append(("in", pairs))
                if self.keep_cache:
                    cache_ref.copy_between(self.k_cache, self.v_cache, self.k_host, self.v_host,
                                           pairs)
            elif kind == "prefill":
                sids = [x for x, _ in op[1]]
                cu = np.concatenate([[0], np.cumsum([n for _, n in op[1]])]).astype(np.int32)
                bt, lens = self.tables(sids)
                res["block_tables"], res["seq_lens"] = bt, lens
                if decode and self.keep_cache:
                    res["out"] = attn.paged_prefill(st.q, self.k_cache, self.v_cache, bt, lens,
                                                    cu, self.shape.scale, n_threads=n_threads,
                                                    sel=sel)
            elif kind == "decode":
                sids = list(op[1])
                bt, lens = self.tables(sids)
                res["decode_seqs"] = sids
                res["block_tables"] = bt
                res["seq_lens"] = lens
                if decode and self.keep_cache:
                    res["out"] = attn.paged_decode(st.q, self.k_cache, self.v_cache, bt, lens,
                                                   self.shape.scale, sel=sel, n_threads=n_threads)
            else:
                raise ValueError(op)
        return res
