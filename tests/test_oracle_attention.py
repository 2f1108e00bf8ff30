"""Pins for the fp64 attention oracle (oracle/attn_ref.c, oracle/attn.py).

Each test pins the oracle to something other than itself: the pages' scalar
worked example, closed forms, brute force over contiguous K/V, torch's SDPA in
float64, and every bit pattern of the storage formats."""
import math

import numpy as np
import pytest
import torch

from conftest import golden
from oracle import attn, cache_ref
from oracle.alloc_ref import RefAllocator

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _caches(nb, hkv, bs, d, dtype, fill=0.0):
    k = torch.full((nb, hkv, bs, d), fill, dtype=DT[dtype])
    v = torch.full((nb, hkv, bs, d), fill, dtype=DT[dtype])
    return k, v


def _place(kc, vc, table, K, V, g=0):
    """Write logical rows K/V [L, D] of KV head g through ``table``, by hand."""
    bs = kc.shape[2]
    for t in range(K.shape[0]):
        kc[table[t // bs], g, t % bs] = K[t]
        vc[table[t // bs], g, t % bs] = V[t]


# ---------------------------------------------------------------- scalar example
def test_scalar_example_both_layouts():
    g = golden("scalar_example.json")
    bs, L, D = g["block_size"], g["length"], g["head_dim"]
    q = torch.full((1, 1, D), g["query"], dtype=torch.float32)
    outs = []
    for layout in g["layouts"]:
        kc, vc = _caches(8, 1, bs, D, "f32")
        K = torch.full((L, D), g["key"])
        V = torch.tensor(g["values"]).reshape(L, D)
        _place(kc, vc, layout, K, V)
        bt = np.array([layout], np.int32)
        out = attn.paged_decode(q, kc, vc, bt, np.array([L], np.int32), 1.0)
        outs.append(out[0, 0, 0])
    assert outs == [g["expected"]] * len(g["layouts"])


@pytest.mark.parametrize("L", range(1, 17))
def test_scalar_mean_any_length(L):
    # equal weights -> the mean of 1..L = (L+1)/2, across the 4->5 block edge
    bs, D = 4, 64
    q = torch.zeros(1, 1, D); q[0, 0, 0] = 1.0
    kc, vc = _caches(8, 1, bs, D, "f32")
    V = torch.zeros(L, D); V[:, 0] = torch.arange(1, L + 1, dtype=torch.float32)
    table = [7, 2, 5, 0][: -(-L // bs)]
    _place(kc, vc, table, torch.zeros(L, D), V)
    out = attn.paged_decode(q, kc, vc, np.array([table + [0] * (4 - len(table))], np.int32),
                            np.array([L], np.int32), 0.125)
    assert out[0, 0, 0] == (L + 1) / 2
    assert np.all(out[0, 0, 1:] == 0)


# ---------------------------------------------------------------- closed forms
def test_two_token_closed_form_scale_and_sign():
    # x0 = scale*a, x1 = 0 -> out = sigmoid(scale*a) * v0 + (1 - sigmoid) * v1
    D, bs, a, scale = 4, 4, 2.0, 0.5
    q = torch.tensor([[[1.0, 0, 0, 0]]])
    kc, vc = _caches(2, 1, bs, D, "f32")
    K = torch.tensor([[a, 0, 0, 0], [0, 0, 0, 0.0]])
    V = torch.tensor([[1.0, 0, 0, 0], [0, 3.0, 0, 0]])
    _place(kc, vc, [1], K, V)
    out = attn.paged_decode(q, kc, vc, np.array([[1]], np.int32), np.array([2], np.int32), scale)
    w = 1.0 / (1.0 + math.exp(-scale * a))
    assert out[0, 0, 0] == pytest.approx(w, rel=1e-15)
    assert out[0, 0, 1] == pytest.approx(3.0 * (1 - w), rel=1e-15)


def test_gqa_head_map_is_contiguous_groups():
    # Hq 4, Hkv 2 -> heads 0,1 read KV head 0 and heads 2,3 read KV head 1
    D, bs, L = 8, 4, 6
    kc, vc = _caches(4, 2, bs, D, "f32")
    for g, c in ((0, 5.0), (1, -7.0)):
        V = torch.full((L, D), c)
        K = torch.randn(L, D, generator=torch.Generator().manual_seed(g))
        _place(kc, vc, [3, 1], K, V, g=g)
    q = torch.randn(1, 4, D, generator=torch.Generator().manual_seed(9))
    out = attn.paged_decode(q, kc, vc, np.array([[3, 1]], np.int32), np.array([L], np.int32), 0.3)
    np.testing.assert_allclose(out[0, :2], 5.0, rtol=1e-15)
    np.testing.assert_allclose(out[0, 2:], -7.0, rtol=1e-15)


def test_large_logits_do_not_overflow():
    D, bs = 4, 4
    q = torch.tensor([[[100.0, 0, 0, 0]]])
    kc, vc = _caches(2, 1, bs, D, "f32")
    K = torch.tensor([[100.0, 0, 0, 0], [90.0, 0, 0, 0], [-100.0, 0, 0, 0]])
    V = torch.tensor([[1.0, 0, 0, 0], [2.0, 0, 0, 0], [3.0, 0, 0, 0]])
    _place(kc, vc, [0], K, V)
    out = attn.paged_decode(q, kc, vc, np.array([[0]], np.int32), np.array([3], np.int32), 1.0)
    # logits 1e4, 9e3, -1e4: weights 1, e^-1000, 0
    assert out[0, 0, 0] == 1.0


def test_positions_beyond_length_and_empty_sequence():
    D, bs, L = 8, 4, 5
    kc, vc = _caches(4, 1, bs, D, "f32", fill=float("nan"))
    g = torch.Generator().manual_seed(3)
    K, V = torch.randn(L, D, generator=g), torch.randn(L, D, generator=g)
    _place(kc, vc, [2, 0], K, V)
    q = torch.randn(2, 1, D, generator=g)
    out = attn.paged_decode(q, kc, vc, np.array([[2, 0], [1, 3]], np.int32),
                            np.array([L, 0], np.int32), 0.5)
    assert np.isfinite(out[0]).all()
    ref = attn.contiguous_attention(q[0, 0].double().numpy(), K.double().numpy(),
                                    V.double().numpy(), 0.5)
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-13, atol=1e-14)
    assert np.all(out[1] == 0)


def test_bad_table_entry_is_an_error():
    kc, vc = _caches(2, 1, 4, 4, "f32")
    q = torch.zeros(1, 1, 4)
    with pytest.raises(ValueError):
        attn.paged_decode(q, kc, vc, np.array([[5]], np.int32), np.array([2], np.int32), 1.0)


# ---------------------------------------------------------------- brute force
def _random_case(seed, dtype, B, Hq, Hkv, D, bs, maxL, nb=None):
    r = np.random.default_rng(seed)
    lens = r.integers(0, maxL + 1, size=B)
    need = sum(-(-int(L) // bs) for L in lens)
    nb = nb or need + 3
    alloc = RefAllocator(nb, bs, list(r.permutation(nb)))
    kc, vc = _caches(nb, Hkv, bs, D, dtype, fill=float("nan"))
    g = torch.Generator().manual_seed(seed)
    logical = []
    for s, L in enumerate(lens):
        alloc.add(s)
        slots, _ = alloc.append(s, int(L))
        K = torch.randn(int(L), Hkv, D, generator=g).to(DT[dtype])
        V = torch.randn(int(L), Hkv, D, generator=g).to(DT[dtype])
        cache_ref.reshape_and_cache(K, V, kc, vc, slots)
        logical.append((K, V))
    width = max(1, max(len(alloc.table(s)) for s in range(B)))
    bt = np.zeros((B, width), np.int32)
    for s in range(B):
        t = alloc.table(s); bt[s, :len(t)] = t
    q = torch.randn(B, Hq, D, generator=g).to(DT[dtype])
    return q, kc, vc, bt, lens.astype(np.int32), logical


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_paged_matches_contiguous_bruteforce(seed, dtype):
    r = np.random.default_rng(100 + seed)
    Hkv = int(r.choice([1, 2]))
    G = int(r.choice([1, 2, 4]))
    bs = int(r.choice([4, 8]))
    D = int(r.choice([16, 64]))
    B = int(r.integers(1, 5))
    q, kc, vc, bt, lens, logical = _random_case(seed, dtype, B, Hkv * G, Hkv, D, bs, 40)
    scale = 1.0 / math.sqrt(D)
    out = attn.paged_decode(q, kc, vc, bt, lens, scale)
    for s in range(B):
        K, V = logical[s]
        for h in range(Hkv * G):
            ref = attn.contiguous_attention(attn.decode_storage(q[s, h]),
                                            attn.decode_storage(K[:, h // G]),
                                            attn.decode_storage(V[:, h // G]), scale)
            np.testing.assert_allclose(out[s, h], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("seed", range(4))
def test_bruteforce_matches_torch_sdpa_float64(seed):
    g = torch.Generator().manual_seed(seed)
    L, D = 1 + 17 * seed, 32
    q, K, V = (torch.randn(n, D, generator=g, dtype=torch.float64) for n in (1, L, L))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None, None], K[None, None], V[None, None], scale=0.2)[0, 0, 0].numpy()
    got = attn.contiguous_attention(q[0].numpy(), K.numpy(), V.numpy(), 0.2)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-14)


def test_permutation_invariance_is_exact():
    """The same logical K/V under two placements give identical fp64 outputs."""
    B, Hq, Hkv, D, bs = 3, 4, 2, 32, 4
    lens = [5, 9, 14]
    g = torch.Generator().manual_seed(7)
    data = [(torch.randn(L, Hkv, D, generator=g), torch.randn(L, Hkv, D, generator=g))
            for L in lens]
    q = torch.randn(B, Hq, D, generator=g)
    outs = []
    for order in (list(range(16)), list(np.random.default_rng(1).permutation(16))):
        alloc = RefAllocator(16, bs, order)
        kc, vc = _caches(16, Hkv, bs, D, "f32")
        for s, (K, V) in enumerate(data):
            alloc.add(s)
            slots, _ = alloc.append(s, lens[s])
            cache_ref.reshape_and_cache(K, V, kc, vc, slots)
        bt = np.zeros((B, 4), np.int32)
        for s in range(B):
            t = alloc.table(s); bt[s, :len(t)] = t
        outs.append((attn.paged_decode(q, kc, vc, bt, np.array(lens, np.int32), 0.25), bt))
    assert not np.array_equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][0], outs[1][0])


def test_selection_matches_full():
    q, kc, vc, bt, lens, _ = _random_case(5, "bf16", 4, 8, 2, 64, 8, 60)
    full = attn.paged_decode(q, kc, vc, bt, lens, 0.125)
    sel = [(3, 7), (0, 0), (2, 5), (1, 1)]
    part = attn.paged_decode(q, kc, vc, bt, lens, 0.125, sel=sel)
    for i, (s, h) in enumerate(sel):
        assert np.array_equal(part[i], full[s, h])


# ---------------------------------------------------------------- split merge
@pytest.mark.parametrize("seed", range(6))
def test_partial_merge_equals_whole(seed):
    r = np.random.default_rng(seed)
    L, D = int(r.integers(1, 300)), 16
    x = r.normal(size=L) * (1 + 10 * seed)
    V = r.normal(size=(L, D))
    cuts = sorted(set(r.integers(0, L + 1, size=int(r.integers(0, 6))).tolist()) | {0, L})
    states = [attn.partial_state(x[a:b], V[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    states.append(attn.partial_state(x[:0], V[:0]))        # an empty range
    w = np.exp(x - x.max())
    np.testing.assert_allclose(attn.merge_partials(states), (w @ V) / w.sum(),
                               rtol=1e-12, atol=1e-13)
    assert np.all(attn.merge_partials([attn.partial_state(x[:0], V[:0])]) == 0)


# ---------------------------------------------------------------- storage formats
def test_f16_decoder_every_bit_pattern(oracle_lib):
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle_lib.attn_ref_decode_value(2, bits.ctypes.data, i)
                    for i in range(1 << 16)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.float16)
    assert np.array_equal(attn.decode_storage(t)[ok], ref[ok])


def test_bf16_decoder_every_bit_pattern(oracle_lib):
    bits = np.arange(1 << 16, dtype=np.uint16)
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    ref = t.to(torch.float64).numpy()
    got = np.array([oracle_lib.attn_ref_decode_value(1, bits.ctypes.data, i)
                    for i in range(1 << 16)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(attn.decode_storage(t)[ok], ref[ok])


def test_f32_decoder(oracle_lib):
    x = np.random.default_rng(0).normal(size=1000).astype(np.float32) * 1e3
    got = np.array([oracle_lib.attn_ref_decode_value(0, x.ctypes.data, i) for i in range(1000)])
    assert np.array_equal(got, x.astype(np.float64))
