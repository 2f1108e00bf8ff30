"""Parity driver: one workload through the oracle and through the CUDA path,
step by step, on the same seeded inputs.  Test helper only."""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

from oracle.run import OracleRun

TOL = {"f32": 1e-5, "bf16": 3e-3, "f16": 3e-3}


def sample_pairs(b: int, hq: int, n: int, seed: int) -> List[Tuple[int, int]]:
    """n distinct (batch index, head) pairs, always including the corners."""
    r = np.random.default_rng(seed)
    pairs = {(0, 0), (b - 1, hq - 1)}
    while len(pairs) < min(n, b * hq):
        pairs.add((int(r.integers(b)), int(r.integers(hq))))
    return sorted(pairs)


def run_parity(wl, table_width: int, sample: Optional[int] = None, max_steps: Optional[int] = None,
               partition_size: int = 0, variant: int = 0, compare_cache: bool = False,
               check_slots: bool = True, prefill_variant: int = 0):
    """Returns a list of per-decode max-abs errors; asserts slots and pairs
    are bit-exact (and the caches too, when ``compare_cache``)."""
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    sh = wl.shape
    orc = OracleRun(sh)
    gpu = PagedKVRunner.for_shape(sh, table_width, partition_size=partition_size,
                                  variant=variant, prefill_variant=prefill_variant)
    errs = []
    for i, st in enumerate(wl.steps):
        if max_steps is not None and i >= max_steps:
            break
        sel = None
        if sample and st.q is not None:
            sel = sample_pairs(st.q.shape[0], sh.num_heads, sample, 1000 + i)
        ref = orc.step(st, sel=sel)
        acts = gpu.plan(st.ops)
        if check_slots:
            slots = [int(x) for a in acts if a.kind == "write" for x in a.slots]
            pairs = [tuple(int(y) for y in p) for a in acts if a.kind == "write" for p in a.pairs]
            assert slots == ref["slots"], f"step {i}: slots differ"
            assert pairs == ref["pairs"], f"step {i}: copy pairs differ"
        gpu.upload(acts)
        dev = lambda t: None if t is None else t.cuda()
        out = gpu.execute(acts, dev(st.k_new), dev(st.v_new), dev(st.q))
        if compare_cache:
            torch.cuda.synchronize()
            assert torch.equal(gpu.k_cache.cpu().view(torch.int16 if sh.dtype != "f32" else torch.int32),
                               orc.k_cache.view(torch.int16 if sh.dtype != "f32" else torch.int32))
            assert torch.equal(gpu.v_cache.cpu().view(torch.int16 if sh.dtype != "f32" else torch.int32),
                               orc.v_cache.view(torch.int16 if sh.dtype != "f32" else torch.int32))
        if ref["out"] is not None:
            got = out.double().cpu().numpy()
            if sel is not None:
                got = np.stack([got[s, h] for s, h in sel])
            assert np.isfinite(got).all(), f"step {i}: non-finite output"
            errs.append(float(np.abs(got - ref["out"]).max()))
    return errs, gpu, orc
