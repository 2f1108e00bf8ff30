"""Pins for the host cache updates (oracle/cache_ref.py) and the oracle's
workload walker (oracle/run.py)."""
import numpy as np
import torch

from oracle import attn, cache_ref
from oracle.alloc_ref import RefAllocator
from oracle.run import OracleRun
import workloads


def test_scatter_round_trips_through_the_table():
    bs, Hkv, D, nb = 4, 2, 8, 12
    alloc = RefAllocator(nb, bs, list(np.random.default_rng(0).permutation(nb)))
    kc = torch.zeros(nb, Hkv, bs, D); vc = torch.zeros(nb, Hkv, bs, D)
    g = torch.Generator().manual_seed(0)
    rows = {}
    for s, L in enumerate([5, 9, 14]):
        alloc.add(s)
        slots, _ = alloc.append(s, L)
        K, V = torch.randn(L, Hkv, D, generator=g), torch.randn(L, Hkv, D, generator=g)
        cache_ref.reshape_and_cache(K, V, kc, vc, slots)
        rows[s] = (K, V)
    for s, (K, V) in rows.items():
        for h in range(Hkv):
            got = attn.gather_logical(kc.double().numpy(), alloc.table(s), K.shape[0], h)
            assert np.array_equal(got, K[:, h].double().numpy())
            got = attn.gather_logical(vc.double().numpy(), alloc.table(s), V.shape[0], h)
            assert np.array_equal(got, V[:, h].double().numpy())


def test_negative_slot_writes_nothing():
    kc = torch.zeros(2, 1, 4, 4); vc = torch.zeros(2, 1, 4, 4)
    k = torch.ones(3, 1, 4); v = 2 * torch.ones(3, 1, 4)
    cache_ref.reshape_and_cache(k, v, kc, vc, [-1, 5, -1])
    assert kc.sum() == 4 and vc.sum() == 8
    assert torch.all(kc[1, 0, 1] == 1) and torch.all(vc[1, 0, 1] == 2)


def test_copy_blocks_uses_the_cache_before_the_call():
    kc = torch.arange(4 * 2 * 2 * 2, dtype=torch.float32).reshape(4, 2, 2, 2)
    vc = -kc.clone()
    k0, v0 = kc.clone(), vc.clone()
    # block 1 is both a destination and (for the second pair) a source
    cache_ref.copy_blocks(kc, vc, [(0, 1), (1, 3)])
    assert torch.equal(kc[1], k0[0]) and torch.equal(kc[3], k0[1])
    assert torch.equal(vc[1], v0[0]) and torch.equal(vc[3], v0[1])
    assert torch.equal(kc[0], k0[0]) and torch.equal(kc[2], k0[2])


def test_tiny_workload_walk():
    wl = workloads.tiny()
    run = OracleRun(wl.shape)
    steps = list(wl.steps)
    r0 = run.step(steps[0])
    assert r0["out"].shape == (3, 2, 64)
    # decode over 5/9/14 tokens uses 2+3+4 blocks of the seeded permutation
    assert run.alloc.stats()["used_blocks"] == 9
    order = list(wl.shape.free_order)
    assert [run.alloc.table(s) for s in range(3)] == [order[0:2], order[2:5], order[5:9]]
    r1 = run.step(steps[1])
    assert run.alloc.stats()["used_blocks"] == 9       # 6/10/15 still fit
    assert list(r1["seq_lens"]) == [6, 10, 15]
    # the appended token of sequence 0 sits at position 5 -> block 1, offset 1
    assert r1["slots"][0] == order[1] * 4 + 1
    # brute force over the logical rows
    K0 = torch.cat([steps[0].k_new[0:5], steps[1].k_new[0:1]])
    V0 = torch.cat([steps[0].v_new[0:5], steps[1].v_new[0:1]])
    for h in range(2):
        ref = attn.contiguous_attention(steps[1].q[0, h].double().numpy(),
                                        K0[:, 0].double().numpy(), V0[:, 0].double().numpy(),
                                        1 / 8)
        np.testing.assert_allclose(r1["out"][0, h], ref, rtol=1e-12, atol=1e-13)


def test_workload_values_are_seeded_and_rounded():
    a = workloads.normal(5, (1, 2), (3, 4), "bf16")
    b = workloads.normal(5, (1, 2), (3, 4), "bf16")
    c = workloads.normal(5, (1, 3), (3, 4), "bf16")
    assert torch.equal(a, b) and not torch.equal(a, c)
    f = workloads.normal(5, (1, 2), (3, 4), "f32")
    assert torch.equal(f.to(torch.bfloat16), a)
    # chunking does not depend on the thread pool: a large draw's head equals
    # the same key drawn small (the first chunk is shared)
    big = workloads.normal(5, (9,), (1 << 23,), "f32")
    small = workloads.normal(5, (9,), (1000,), "f32")
    assert torch.equal(big[:1000], small)


def test_copy_between_moves_each_source_block_onto_its_destination():
    """The swap copy (sanketn26 "PagedAttention", "What this does not solve":
    a preempted request's blocks leave for host memory and come back).  Pairs
    are (source block, destination block); the expected caches are written out
    value by value, so a swapped orientation, a copy of the wrong cache or a
    touched bystander block fails."""
    # source caches: 3 blocks of [Hkv 1][bs 2][D 2]; block b holds 10*b + i
    src_k = torch.tensor([[[[0., 1.], [2., 3.]]],
                          [[[10., 11.], [12., 13.]]],
                          [[[20., 21.], [22., 23.]]]])
    src_v = -src_k - 100.
    # destination caches: 4 blocks, every value 7 (K) and 9 (V)
    dst_k = torch.full((4, 1, 2, 2), 7.)
    dst_v = torch.full((4, 1, 2, 2), 9.)
    src_k0, src_v0 = src_k.clone(), src_v.clone()
    # source 2 -> destination 0, source 0 -> destination 3; source 1 unused
    cache_ref.copy_between(dst_k, dst_v, src_k, src_v, [(2, 0), (0, 3)])
    exp_k = torch.tensor([[[[20., 21.], [22., 23.]]],
                          [[[7., 7.], [7., 7.]]],
                          [[[7., 7.], [7., 7.]]],
                          [[[0., 1.], [2., 3.]]]])
    exp_v = torch.tensor([[[[-120., -121.], [-122., -123.]]],
                          [[[9., 9.], [9., 9.]]],
                          [[[9., 9.], [9., 9.]]],
                          [[[-100., -101.], [-102., -103.]]]])
    assert torch.equal(dst_k, exp_k)
    assert torch.equal(dst_v, exp_v)
    # the source side is read only
    assert torch.equal(src_k, src_k0) and torch.equal(src_v, src_v0)


def test_copy_between_round_trip_restores_the_blocks_in_new_places():
    """Out to a host pool and back in to different device blocks: the
    sequence's rows reappear bit for bit at the new places (16-bit storage,
    so the copy must be bitwise, not a value conversion)."""
    g = torch.Generator().manual_seed(3)
    dev_k = torch.randn(6, 2, 4, 8, generator=g).to(torch.bfloat16)
    dev_v = torch.randn(6, 2, 4, 8, generator=g).to(torch.bfloat16)
    host_k = torch.zeros(3, 2, 4, 8, dtype=torch.bfloat16)
    host_v = torch.zeros(3, 2, 4, 8, dtype=torch.bfloat16)
    orig_k, orig_v = dev_k.clone(), dev_v.clone()
    cache_ref.copy_between(host_k, host_v, dev_k, dev_v, [(4, 0), (1, 1), (5, 2)])
    assert torch.equal(host_k[0].view(torch.int16), orig_k[4].view(torch.int16))
    assert torch.equal(host_v[2].view(torch.int16), orig_v[5].view(torch.int16))
    cache_ref.copy_between(dev_k, dev_v, host_k, host_v, [(0, 0), (1, 2), (2, 3)])
    for new, old in ((0, 4), (2, 1), (3, 5)):
        assert torch.equal(dev_k[new].view(torch.int16), orig_k[old].view(torch.int16))
        assert torch.equal(dev_v[new].view(torch.int16), orig_v[old].view(torch.int16))
    # blocks 1, 4 and 5 were not destinations of the way back in
    for b in (1, 4, 5):
        assert torch.equal(dev_k[b].view(torch.int16), orig_k[b].view(torch.int16))
