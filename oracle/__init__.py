"""Oracle for the paged-KV decode path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct CPU code that states what the path computes:

* ``alloc_ref``  -- the block allocator (free list, refcounts, fork, free,
  copy-on-write on append to a shared block) as a Python model;
* ``attn_ref.c`` -- single-query attention over a block-paged KV cache in
  fp64 C: every token is gathered through the block table and the softmax is
  the exact two-pass one (max, then exp-sum), no online recurrence; and the
  same for several new tokens per sequence under a causal mask (chunked
  prefill);
* ``attn``       -- ctypes entry to ``attn_ref.c``, a numpy fp64 brute force
  over contiguous (already gathered) K/V, the split-partial merge, and the
  storage-dtype decoders;
* ``cache_ref``  -- the KV append scatter and the block copy on host tensors;
* ``run``        -- walks a ``workloads`` event list through the pieces above.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import or run anything here.  The product package never does, and this
package imports nothing from the product: the two share only the seeded input
generators in ``workloads``.

Sources: the three PagedAttention pages -- paweldubiel.com "PagedAttention"
(block table, four-position blocks, the scalar worked example); sanketn26
"PagedAttention -- grow the allocation with the sequence" (logical vs physical
blocks, capacity arithmetic, copy-on-write ownership, release on completion);
mbrenndoerfer.com "Paged Attention > Summary" (gather through the block table,
one partial block per sequence, copy-on-write for beams).

Every function is pinned by a ``-m "not gpu"`` test (tests/test_oracle_*.py)
to values the pages print, closed forms, brute force or a library routine.
"""
