"""Seeded synthetic inputs for the paged-KV decode path.

This module is the only code shared by the oracle (``oracle/``) and the CUDA
path (``paged_kv_cache_347_b200``).  It draws random numbers and lays out the
order of sequence events (add, append, fork, free, decode); it holds none of
the method's arithmetic: no slot or block-table computation, no attention, no
cache scatter or copy.  Each side runs the same event list through its own
allocator and its own attention.

Values are N(0, 1) drawn in float32 from numpy's PCG64 and rounded to the
storage dtype with torch's round-to-nearest-even ``.to()``.  Every tensor is
drawn from its own key, in fixed 4 Mi-element chunks, each chunk seeded by
``SeedSequence(entropy=seed, spawn_key=key + (chunk,))``, so a tensor does not
depend on thread count or on the order in which other tensors are drawn.

The five workloads follow the shapes named in the PagedAttention pages'
examples (sanketn26 "PagedAttention -- grow the allocation with the sequence",
"Work the capacity arithmetic": lengths 5/9/14, four-position blocks) and the
decode shapes of a Llama-8B-like model (32/8 heads, head_dim 128), a 32k
long-context batch, a beam-search prefix-sharing batch and a
continuous-batching mix.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Iterator, List, Optional, Sequence, Tuple

import numpy as np
import torch

__all__ = [
    "DTYPES", "DTYPE_CODES", "normal", "permutation", "Shape", "Op", "Step",
    "Workload", "tiny", "llama", "long_context", "beam", "mix", "custom",
    "WORKLOADS", "get",
]

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
# codes of the C ABI's pa_dtype enum
DTYPE_CODES = {"f32": 0, "bf16": 1, "f16": 2}

_CHUNK = 1 << 22


def normal(seed: int, key: Sequence[int], shape: Sequence[int], dtype: str) -> torch.Tensor:
    """N(0,1) float32 draws rounded to ``dtype``; a contiguous CPU tensor."""
    n = int(np.prod(shape, dtype=np.int64)) if len(shape) else 1
    buf = np.empty(n, np.float32)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)

    def fill(i: int) -> None:
        ss = np.random.SeedSequence(entropy=seed, spawn_key=tuple(key) + (i,))
        g = np.random.Generator(np.random.PCG64(ss))
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        if hi > lo:
            g.standard_normal(out=buf[lo:hi], dtype=np.float32)

    if nchunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(8) as ex:
            list(ex.map(fill, range(nchunks)))
    t = torch.from_numpy(buf).reshape(tuple(shape))
    return t.to(DTYPES[dtype]).contiguous()


def rng_for(seed: int, key: Sequence[int]) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=tuple(key))))


def permutation(seed: int, n: int) -> np.ndarray:
    """Seeded free-list order: a permutation of 0..n-1 (int32)."""
    return rng_for(seed, (1,)).permutation(n).astype(np.int32)


@dataclass
class Shape:
    name: str
    num_heads: int          # Hq
    num_kv_heads: int       # Hkv
    head_dim: int           # D
    dtype: str              # "f32" | "bf16" | "f16"
    block_size: int         # bs
    num_blocks: int         # NB, pool size in blocks
    seed: int
    free_order: Optional[np.ndarray] = None   # None: identity 0..NB-1
    scale: float = 0.0      # softmax scale; 0 means 1/sqrt(D)

    def __post_init__(self) -> None:
        if self.scale == 0.0:
            self.scale = 1.0 / math.sqrt(self.head_dim)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


# An event on the sequences, applied in list order.
#   ("add", sid) ("append", sid, n) ("fork", parent, child) ("free", sid)
#   ("decode", [sid, ...])
#   ("admit", sid, token_ids)        new sequence with token ids (prefix cache)
#   ("append_tokens", sid, token_ids)
#   ("host_pool", n_blocks) ("swap_out", sid) ("swap_in", sid)
#   ("prefill", [(sid, n), ...])     causal attention of each sid's last n
#                                    tokens; the step's q holds their rows
Op = Tuple


@dataclass
class Step:
    """One batch of events.

    ``k_new``/``v_new`` hold the K/V rows of every ``append`` op of the step,
    concatenated in op order, shape [N, Hkv, D]; ``q`` holds one query row per
    sequence of the step's single ``decode`` op (in that op's order), shape
    [b, Hq, D].  Either may be None when the step has no such op.
    """
    ops: List[Op]
    k_new: Optional[torch.Tensor] = None
    v_new: Optional[torch.Tensor] = None
    q: Optional[torch.Tensor] = None
    tag: str = ""

    @property
    def n_new_tokens(self) -> int:
        """K/V rows the step carries: every appended token, and every token of
        an admitted sequence (the prefix cache may make some rows unused)."""
        n = 0
        for op in self.ops:
            if op[0] == "append":
                n += op[2]
            elif op[0] in ("admit", "append_tokens"):
                n += len(op[2])
        return n

    @property
    def decode_seqs(self) -> List[int]:
        for op in self.ops:
            if op[0] == "decode":
                return list(op[1])
        return []


@dataclass
class Workload:
    shape: Shape
    steps: Iterator[Step]
    description: str = ""
    meta: dict = field(default_factory=dict)


def _kv(shape: Shape, key: Tuple[int, ...], n: int) -> Tuple[torch.Tensor, torch.Tensor]:
    dims = (n, shape.num_kv_heads, shape.head_dim)
    return normal(shape.seed, key + (0,), dims, shape.dtype), normal(shape.seed, key + (1,), dims, shape.dtype)


def _q(shape: Shape, key: Tuple[int, ...], b: int) -> torch.Tensor:
    return normal(shape.seed, key + (2,), (b, shape.num_heads, shape.head_dim), shape.dtype)


def _prefill_step(shape: Shape, lens: Sequence[int], sids: Sequence[int], key, decode: bool) -> Step:
    ops: List[Op] = [("add", s) for s in sids]
    ops += [("append", s, int(n)) for s, n in zip(sids, lens)]
    k, v = _kv(shape, key, int(sum(lens)))
    q = None
    if decode:
        ops.append(("decode", list(sids)))
        q = _q(shape, key, len(sids))
    return Step(ops, k, v, q, tag="prefill")


def _decode_step(shape: Shape, sids: Sequence[int], key, tag="decode") -> Step:
    ops: List[Op] = [("append", s, 1) for s in sids]
    ops.append(("decode", list(sids)))
    k, v = _kv(shape, key, len(sids))
    return Step(ops, k, v, _q(shape, key, len(sids)), tag=tag)


def tiny(seed: int = 0) -> Workload:
    """Three sequences of lengths 5, 9, 14 at block size 4 in a 16-block pool,
    2 query heads / 1 KV head, head_dim 64, fp32; one decode over the prefill,
    then one appended token per sequence and a second decode."""
    sh = Shape("tiny", 2, 1, 64, "f32", 4, 16, seed)
    sh.free_order = permutation(seed, 16)
    sh.scale = 1.0 / 8.0
    lens = [5, 9, 14]

    def gen():
        yield _prefill_step(sh, lens, [0, 1, 2], (10,), decode=True)
        yield _decode_step(sh, [0, 1, 2], (11,))

    return Workload(sh, gen(), "tiny: lens 5/9/14, bs 4, NB 16, 2/1 heads, D 64, fp32",
                    {"lens": lens})


def llama(seed: int = 1, steps: int = 1, batch: int = 32, lo: int = 512, hi: int = 4096,
          num_blocks: int = 16384) -> Workload:
    """Llama-8B-shaped decode: batch 32, 32/8 heads, D 128, bf16, bs 16,
    lengths uniform in [512, 4096], 16k-block pool in a seeded permutation.
    The prefill writes L_s - 1 tokens; each decode step appends one token per
    sequence and attends over the grown context (the first step over L_s)."""
    sh = Shape("llama8b", 32, 8, 128, "bf16", 16, num_blocks, seed)
    sh.free_order = permutation(seed, num_blocks)
    lens = rng_for(seed, (2,)).integers(lo, hi, size=batch, endpoint=True).astype(np.int64)
    sids = list(range(batch))

    def gen():
        yield _prefill_step(sh, [int(x) - 1 for x in lens], sids, (10,), decode=False)
        for t in range(steps):
            yield _decode_step(sh, sids, (20, t))

    return Workload(sh, gen(), "llama8b-shaped decode", {"lens": lens.tolist()})


def long_context(seed: int = 2, steps: int = 1, batch: int = 8, seq_len: int = 32768,
                 num_blocks: int = 32768) -> Workload:
    """Long context: batch 8, 64/8 heads, D 128, bf16, bs 16, every sequence
    reaching ``seq_len`` tokens at the last decode step.  The prefill writes
    ``seq_len - steps`` tokens; each step appends one token per sequence and
    decodes.  Pool of 32768 blocks in a seeded permutation (blocks scattered)."""
    sh = Shape("long32k", 64, 8, 128, "bf16", 16, num_blocks, seed)
    sh.free_order = permutation(seed, num_blocks)
    sids = list(range(batch))
    pre = seq_len - steps

    def gen():
        yield _prefill_step(sh, [pre] * batch, sids, (10,), decode=False)
        for t in range(steps):
            yield _decode_step(sh, sids, (20, t))

    return Workload(sh, gen(), "long context 32k", {"lens": [seq_len] * batch, "prefill": pre})


def beam(seed: int = 3, steps: int = 256, groups: int = 4, beams: int = 4, prefix: int = 2050,
         num_blocks: int = 4096) -> Workload:
    """Prefix sharing / beam search: ``groups`` prompts of ``prefix`` tokens,
    each forked into ``beams`` sequences sharing the prefix blocks, then
    ``steps`` decode steps in which every beam appends its own token.
    32/8 heads, D 128, fp16, bs 16, 4096-block pool in a seeded permutation.
    Sequence ids: group g, beam b -> g*beams + b; beam 0 is the prompt."""
    sh = Shape("beam", 32, 8, 128, "f16", 16, num_blocks, seed)
    sh.free_order = permutation(seed, num_blocks)
    roots = [g * beams for g in range(groups)]
    all_sids = [g * beams + b for g in range(groups) for b in range(beams)]

    def gen():
        st = _prefill_step(sh, [prefix] * groups, roots, (10,), decode=False)
        for g in range(groups):
            for b in range(1, beams):
                st.ops.append(("fork", g * beams, g * beams + b))
        yield st
        for t in range(steps):
            yield _decode_step(sh, all_sids, (20, t), tag="cow" if t == 0 else "decode")

    return Workload(sh, gen(), "prefix sharing / beam search",
                    {"groups": groups, "beams": beams, "prefix": prefix})


def mix(seed: int = 4, block_size: int = 16, steps: int = 32, batch: int = 256, lo: int = 16,
        hi: int = 8192, finish_frac: float = 0.1, admit_len: int = 128,
        pool_slots: int = 524288) -> Workload:
    """Continuous-batching mix: 256 sequences with lengths log-uniform in
    [16, 8192], 32/8 heads, D 128, bf16.  Each step appends one token to every
    live sequence and decodes the batch; then 10% of the sequences (drawn with
    the seeded generator) finish and free their blocks, and as many new
    sequences are admitted with 128-token prefills.  Pool of ``pool_slots``
    token slots, i.e. pool_slots / block_size blocks, in a seeded permutation."""
    nb = pool_slots // block_size
    sh = Shape(f"mix_bs{block_size}", 32, 8, 128, "bf16", block_size, nb, seed)
    sh.free_order = permutation(seed, nb)
    r = rng_for(seed, (2,))
    lens = np.rint(np.exp(r.uniform(math.log(lo), math.log(hi), size=batch))).astype(np.int64)
    lens = np.clip(lens, lo, hi)
    choose = rng_for(seed, (3,))
    n_finish = int(math.floor(finish_frac * batch))

    def gen():
        live = list(range(batch))
        next_id = batch
        yield _prefill_step(sh, [int(x) - 1 for x in lens], live, (10,), decode=False)
        for t in range(steps):
            st = _decode_step(sh, live, (20, t))
            fin_idx = sorted(choose.choice(len(live), size=n_finish, replace=False).tolist())
            fin = [live[i] for i in fin_idx]
            new = list(range(next_id, next_id + n_finish))
            next_id += n_finish
            st.ops += [("free", s) for s in fin]
            st.ops += [("add", s) for s in new]
            st.ops += [("append", s, admit_len) for s in new]
            k2, v2 = _kv(sh, (30, t), admit_len * n_finish)
            st.k_new = torch.cat([st.k_new, k2])
            st.v_new = torch.cat([st.v_new, v2])
            # the admitted sequences take the finished ones' batch positions
            for i, s in zip(fin_idx, new):
                live[i] = s
            yield st

    return Workload(sh, gen(), f"continuous-batching mix bs {block_size}",
                    {"lens": lens.tolist(), "finish": n_finish, "admit": admit_len})


def custom(name: str, lens: Sequence[int], num_heads: int, num_kv_heads: int, head_dim: int,
           dtype: str, block_size: int, num_blocks: int, seed: int, steps: int = 1,
           permute: bool = True, scale: float = 0.0) -> Workload:
    """Any shape: prefill ``L_s - steps`` tokens per sequence (>= 0), then
    ``steps`` decode steps appending one token each (a sequence of length 0
    with steps == 0 decodes an empty context)."""
    sh = Shape(name, num_heads, num_kv_heads, head_dim, dtype, block_size, num_blocks, seed,
               scale=scale)
    if permute:
        sh.free_order = permutation(seed, num_blocks)
    sids = list(range(len(lens)))

    def gen():
        pre = [max(0, int(x) - steps) for x in lens]
        yield _prefill_step(sh, pre, sids, (10,), decode=(steps == 0))
        for t in range(steps):
            yield _decode_step(sh, sids, (20, t))

    return Workload(sh, gen(), name, {"lens": list(lens)})


def prefix_share(seed: int = 5, requests: int = 16, prompt: int = 1000, suffix_lo: int = 1,
                 suffix_hi: int = 200, steps: int = 2, block_size: int = 16,
                 num_blocks: int = 4096, vocab: int = 32000) -> Workload:
    """Prefix caching: ``requests`` sequences share a ``prompt``-token system
    prompt (same token ids, hence the same K/V rows) followed by their own
    suffix; they are admitted one by one with their token ids ("admit"), then
    decode ``steps`` tokens each ("append_tokens" + "decode").  32/8 heads,
    D 128, bf16.  The K/V rows of an admit op cover all of its tokens; the
    runner writes only the ones the prefix cache does not already hold."""
    sh = Shape("prefix", 32, 8, 128, "bf16", block_size, num_blocks, seed)
    sh.free_order = permutation(seed, num_blocks)
    r = rng_for(seed, (5,))
    sys_ids = r.integers(0, vocab, size=prompt).tolist()
    sfx = r.integers(suffix_lo, suffix_hi, size=requests, endpoint=True).tolist()
    pk, pv = _kv(sh, (40,), prompt)
    sids = list(range(requests))

    def gen():
        ops: List[Op] = []
        ks, vs = [], []
        for i in sids:
            ids = sys_ids + r.integers(0, vocab, size=sfx[i]).tolist()
            ops.append(("admit", i, ids))
            k2, v2 = _kv(sh, (41, i), sfx[i])
            ks += [pk, k2]
            vs += [pv, v2]
        yield Step(ops, torch.cat(ks), torch.cat(vs), tag="admit")
        for t in range(steps):
            ops = [("append_tokens", i, [int(r.integers(0, vocab))]) for i in sids]
            ops.append(("decode", sids))
            k, v = _kv(sh, (20, t), len(sids))
            yield Step(ops, k, v, _q(sh, (20, t), len(sids)), tag="decode")

    return Workload(sh, gen(), "prefix sharing with a cached system prompt",
                    {"prompt": prompt, "suffix": sfx})


def preempt(seed: int = 6, batch: int = 8, lo: int = 200, hi: int = 3000, steps: int = 6,
            victim: int = 0, out_step: int = 1, in_step: int = 4, host_blocks: int = 512,
            block_size: int = 16, num_blocks: int = 2048) -> Workload:
    """Preemption by swap: a batch decodes; at ``out_step`` one sequence is
    swapped out to host blocks and a newcomer is admitted into the freed
    device blocks; at ``in_step`` the newcomer finishes and the preempted
    sequence is swapped back in and decodes on.  32/8 heads, D 128, bf16."""
    sh = Shape("preempt", 32, 8, 128, "bf16", block_size, num_blocks, seed)
    sh.free_order = permutation(seed, num_blocks)
    lens = rng_for(seed, (2,)).integers(lo, hi, size=batch, endpoint=True).tolist()
    newcomer = batch

    def gen():
        st = _prefill_step(sh, [int(x) - 1 for x in lens], list(range(batch)), (10,), decode=False)
        st.ops.insert(0, ("host_pool", host_blocks))
        yield st
        live = list(range(batch))
        for t in range(steps):
            pre: List[Op] = []
            k0 = v0 = None
            if t == out_step:
                pre = [("swap_out", victim), ("add", newcomer), ("append", newcomer, lens[victim])]
                live = [s for s in live if s != victim] + [newcomer]
                k0, v0 = _kv(sh, (50,), lens[victim])
            elif t == in_step:
                pre = [("free", newcomer), ("swap_in", victim)]
                live = [s for s in live if s != newcomer] + [victim]
            st = _decode_step(sh, live, (20, t))
            st.ops = pre + st.ops
            if k0 is not None:
                st.k_new = torch.cat([k0, st.k_new])
                st.v_new = torch.cat([v0, st.v_new])
            yield st

    return Workload(sh, gen(), "preemption by swap", {"lens": lens, "victim": victim})


def chunked_prefill(seed: int = 7, batch: int = 4, ctx_lo: int = 0, ctx_hi: int = 600,
                    chunk_lo: int = 1, chunk_hi: int = 300, num_heads: int = 32,
                    num_kv_heads: int = 8, head_dim: int = 128, dtype: str = "bf16",
                    block_size: int = 16, num_blocks: int = 1024, chunks: int = 1) -> Workload:
    """Multi-token attention over the paged cache: each sequence has a
    context of U[ctx_lo, ctx_hi] tokens, then ``chunks`` times appends a chunk
    of U[chunk_lo, chunk_hi] tokens and attends them causally ("prefill",
    [(sid, n), ...]); the chunk's queries are packed in op order."""
    sh = Shape("chunked", num_heads, num_kv_heads, head_dim, dtype, block_size, num_blocks, seed)
    sh.free_order = permutation(seed, num_blocks)
    r = rng_for(seed, (6,))
    ctx = r.integers(ctx_lo, ctx_hi, size=batch, endpoint=True).tolist()
    sids = list(range(batch))

    def gen():
        yield _prefill_step(sh, ctx, sids, (10,), decode=False)
        for c in range(chunks):
            n = r.integers(chunk_lo, chunk_hi, size=batch, endpoint=True).tolist()
            ops: List[Op] = [("append", s, int(x)) for s, x in zip(sids, n)]
            ops.append(("prefill", [(s, int(x)) for s, x in zip(sids, n)]))
            k, v = _kv(sh, (60, c), int(sum(n)))
            q = normal(sh.seed, (60, c, 2), (int(sum(n)), sh.num_heads, sh.head_dim), sh.dtype)
            yield Step(ops, k, v, q, tag="chunk")

    return Workload(sh, gen(), "chunked prefill", {"ctx": ctx})


WORKLOADS = {
    "tiny": tiny,
    "llama8b": llama,
    "long32k": long_context,
    "beam": beam,
    "mix": mix,
    "prefix": prefix_share,
    "preempt": preempt,
}


def get(name: str, **kw) -> Workload:
    return WORKLOADS[name](**kw)
