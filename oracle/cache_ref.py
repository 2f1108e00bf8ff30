"""Reference KV-cache updates on host tensors -- TEST INFRASTRUCTURE ONLY.

* ``reshape_and_cache``: the append.  The token written for position p of a
  sequence goes to slot ``phys * bs + off`` (paweldubiel.com "PagedAttention",
  "Mechanism and details": a block holds a fixed number of positions, and
  appending never moves the prefix); its K row for KV head h lands at
  ``k_cache[slot // bs, h, slot % bs, :]``, and likewise V.  A negative slot
  means "no write".
* ``copy_blocks``: the copy-on-write block copy (sanketn26 "PagedAttention",
  "Sharing needs ownership rules": make a private copy before changing a
  shared block).  Every listed (src, dst) pair copies the whole physical
  block, all KV heads and positions, of both caches.  The pairs act together
  on the cache as it was before the call.

Caches are CPU tensors [NB, Hkv, bs, D] in the storage dtype; copies are
bitwise.
"""
from __future__ import annotations

from typing import Iterable, Sequence, Tuple

import numpy as np
import torch


def reshape_and_cache(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, slots: Sequence[int]) -> None:
    slots = np.asarray(slots, dtype=np.int64).reshape(-1)
    assert k.shape[0] == slots.shape[0] == v.shape[0]
    keep = slots >= 0
    if not keep.any():
        return
    live = slots[keep]
    assert np.unique(live).shape[0] == live.shape[0], "slots must be distinct"
    bs = k_cache.shape[2]
    assert live.max() < k_cache.shape[0] * bs
    pb = torch.from_numpy(live // bs)
    off = torch.from_numpy(live % bs)
    sel = torch.from_numpy(keep)
    k_cache[pb, :, off, :] = k[sel]
    v_cache[pb, :, off, :] = v[sel]


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor,
                pairs: Iterable[Tuple[int, int]]) -> None:
    pairs = [(int(a), int(b)) for a, b in pairs]
    if not pairs:
        return
    src = torch.tensor([a for a, _ in pairs], dtype=torch.int64)
    dst = torch.tensor([b for _, b in pairs], dtype=torch.int64)
    k_src = k_cache[src].clone()
    v_src = v_cache[src].clone()
    k_cache[dst] = k_src
    v_cache[dst] = v_src


def copy_between(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                 src_v: torch.Tensor, pairs: Iterable[Tuple[int, int]]) -> None:
    """Swap copy: block a of the source caches onto block b of the
    destination caches for each (a, b), bitwise."""
    pairs = [(int(a), int(b)) for a, b in pairs]
    if not pairs:
        return
    src = torch.tensor([a for a, _ in pairs], dtype=torch.int64)
    dst = torch.tensor([b for _, b in pairs], dtype=torch.int64)
    dst_k[dst] = src_k[src]
    dst_v[dst] = src_v[src]
