"""Pins for the chunked-prefill oracle (oracle/attn_ref.c, attn_ref_prefill):
causal attention of several new tokens over the paged cache."""
import math

import numpy as np
import pytest
import torch

from conftest import golden
from oracle import attn, cache_ref
from oracle.alloc_ref import RefAllocator

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def test_running_mean_extends_the_scalar_example():
    """Keys 0, query 1, values 1..5 ([P1] "Text order is not a memory
    address"): a causal chunk of all five positions gives the running means
    1, 1.5, 2, 2.5, 3 -- the last one is the page's 3 -- in both layouts."""
    g = golden("scalar_example.json")
    bs, L, D = g["block_size"], g["length"], 1
    for layout in g["layouts"]:
        kc = torch.zeros(8, 1, bs, D); vc = torch.zeros(8, 1, bs, D)
        for t in range(L):
            vc[layout[t // bs], 0, t % bs, 0] = g["values"][t]
        q = torch.full((L, 1, D), g["query"])
        out = attn.paged_prefill(q, kc, vc, np.array([layout], np.int32),
                                 np.array([L], np.int32), np.array([0, L], np.int32), 1.0)
        assert out[:, 0, 0].tolist() == [(p + 2) / 2 for p in range(L)]
        assert out[-1, 0, 0] == g["expected"]


def _case(seed, dtype, lens, chunks, Hq, Hkv, D, bs):
    r = np.random.default_rng(seed)
    nb = sum(-(-L // bs) for L in lens) + 3
    alloc = RefAllocator(nb, bs, list(r.permutation(nb)))
    kc = torch.full((nb, Hkv, bs, D), float("nan")).to(DT[dtype])
    vc = torch.full((nb, Hkv, bs, D), float("nan")).to(DT[dtype])
    g = torch.Generator().manual_seed(seed)
    logical = []
    for s, L in enumerate(lens):
        alloc.add(s)
        slots, _ = alloc.append(s, L)
        K = torch.randn(L, Hkv, D, generator=g).to(DT[dtype])
        V = torch.randn(L, Hkv, D, generator=g).to(DT[dtype])
        cache_ref.reshape_and_cache(K, V, kc, vc, slots)
        logical.append((K, V))
    W = max(len(alloc.table(s)) for s in range(len(lens)))
    bt = np.zeros((len(lens), W), np.int32)
    for s in range(len(lens)):
        t = alloc.table(s); bt[s, :len(t)] = t
    cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = torch.randn(int(cu[-1]), Hq, D, generator=g).to(DT[dtype])
    return q, kc, vc, bt, np.array(lens, np.int32), cu, logical


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("seed", range(3))
def test_prefill_matches_torch_sdpa_with_causal_mask(dtype, seed):
    lens, chunks = [23, 9, 40], [7, 9, 1]
    Hq, Hkv, D, bs = 4, 2, 16, 4
    q, kc, vc, bt, sl, cu, logical = _case(seed, dtype, lens, chunks, Hq, Hkv, D, bs)
    scale = 0.3
    out = attn.paged_prefill(q, kc, vc, bt, sl, cu, scale)
    G = Hq // Hkv
    for s, (L, n) in enumerate(zip(lens, chunks)):
        K, V = logical[s]
        rows = q[cu[s]:cu[s + 1]]
        pos = torch.arange(L - n, L)[:, None]
        mask = torch.arange(L)[None, :] <= pos           # [n, L]
        for h in range(Hq):
            qh = torch.from_numpy(attn.decode_storage(rows[:, h]))[None, None]
            kh = torch.from_numpy(attn.decode_storage(K[:, h // G]))[None, None]
            vh = torch.from_numpy(attn.decode_storage(V[:, h // G]))[None, None]
            ref = torch.nn.functional.scaled_dot_product_attention(
                qh, kh, vh, attn_mask=mask[None, None], scale=scale)[0, 0].numpy()
            np.testing.assert_allclose(out[cu[s]:cu[s + 1], h], ref, rtol=1e-12, atol=1e-13)


def test_last_row_of_a_chunk_is_the_decode_result():
    lens, chunks = [33, 17], [5, 17]
    q, kc, vc, bt, sl, cu, _ = _case(7, "f32", lens, chunks, 8, 2, 64, 8)
    out = attn.paged_prefill(q, kc, vc, bt, sl, cu, 0.125)
    last = torch.stack([q[cu[s + 1] - 1] for s in range(2)])
    dec = attn.paged_decode(last, kc, vc, bt, sl, 0.125)
    assert np.array_equal(out[cu[1:] - 1], dec)


def test_rows_never_see_later_positions():
    lens, chunks = [20], [6]
    q, kc, vc, bt, sl, cu, _ = _case(3, "f32", lens, chunks, 2, 1, 16, 4)
    base = attn.paged_prefill(q, kc, vc, bt, sl, cu, 0.5)
    # overwrite the K/V of position 17 (row 3 of the chunk sits at position 17)
    blk, off = bt[0][17 // 4], 17 % 4
    kc[blk, :, off] = 100.0; vc[blk, :, off] = -100.0
    moved = attn.paged_prefill(q, kc, vc, bt, sl, cu, 0.5)
    assert np.array_equal(moved[:3], base[:3])           # positions 14, 15, 16
    assert not np.allclose(moved[3:], base[3:])


def test_bad_chunk_is_an_error():
    q, kc, vc, bt, sl, cu, _ = _case(1, "f32", [5], [5], 2, 1, 16, 4)
    with pytest.raises(ValueError):
        attn.paged_prefill(q[:5], kc, vc, bt, np.array([4], np.int32), cu, 1.0)


def test_selected_rows_equal_the_full_computation():
    """attn_ref_prefill_sel computes exactly the listed (row, head) pairs of
    attn_ref_prefill (same per-row loop); an out-of-range pair is an error."""
    import workloads
    from oracle.run import OracleRun
    wl = workloads.chunked_prefill(batch=3, ctx_lo=20, ctx_hi=90, chunk_lo=1, chunk_hi=40,
                                   num_heads=8, num_kv_heads=2, head_dim=64, dtype="bf16",
                                   block_size=8, num_blocks=128)
    o = OracleRun(wl.shape)
    steps = list(wl.steps)
    o.step(steps[0])
    st = steps[1]
    ref = o.step(st)
    ns = [n for op in st.ops if op[0] == "prefill" for _, n in op[1]]
    cu = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    sel = [(0, 0), (5, 3), (int(cu[-1]) - 1, 7), (int(cu[1]), 2)]
    part = attn.paged_prefill(st.q, o.k_cache, o.v_cache, ref["block_tables"], ref["seq_lens"],
                              cu, wl.shape.scale, sel=sel)
    for j, (r, h) in enumerate(sel):
        assert np.array_equal(part[j], ref["out"][r, h])
    with pytest.raises(ValueError):
        attn.paged_prefill(st.q, o.k_cache, o.v_cache, ref["block_tables"], ref["seq_lens"],
                           cu, wl.shape.scale, sel=[(int(cu[-1]), 0)])
