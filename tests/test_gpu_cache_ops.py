"""pa_reshape_and_cache and pa_copy_blocks must be bit-exact against the
oracle's host cache updates (needs a B200)."""
import numpy as np
import pytest
import torch

from oracle import cache_ref
from oracle.alloc_ref import RefAllocator
from oracle.run import OracleRun
from parity import run_parity
import workloads

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
BITS = {"f32": torch.int32, "bf16": torch.int16, "f16": torch.int16}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _rand_bits(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    bits = BITS[dtype]
    lo, hi = (-2 ** 31, 2 ** 31 - 1) if bits == torch.int32 else (-2 ** 15, 2 ** 15 - 1)
    return torch.randint(lo, hi, shape, generator=g, dtype=bits).view(DT[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("D,bs,Hkv", [(64, 4, 1), (128, 16, 8), (128, 32, 2), (64, 8, 3),
                                      (128, 64, 2)])
def test_reshape_and_cache_bit_exact(dtype, D, bs, Hkv):
    from paged_kv_cache_347_b200 import pagedattn as pa
    NB, N = 160, 300
    r = np.random.default_rng(D + bs)
    slots = r.choice(NB * bs, size=N, replace=False).astype(np.int64)
    slots[r.random(N) < 0.1] = -1
    kc = _rand_bits((NB, Hkv, bs, D), dtype, 1)
    vc = _rand_bits((NB, Hkv, bs, D), dtype, 2)
    k = _rand_bits((N, Hkv, D), dtype, 3)
    v = _rand_bits((N, Hkv, D), dtype, 4)
    dk, dv = kc.cuda(), vc.cuda()
    pa.pa_reshape_and_cache(k.cuda(), v.cuda(), dk, dv, torch.from_numpy(slots).cuda())
    # the oracle moves the raw bits (integer views), so NaN payloads survive
    b = BITS[dtype]
    cache_ref.reshape_and_cache(k.view(b), v.view(b), kc.view(b), vc.view(b), slots)
    assert torch.equal(dk.cpu().view(BITS[dtype]), kc.view(BITS[dtype]))
    assert torch.equal(dv.cpu().view(BITS[dtype]), vc.view(BITS[dtype]))


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_copy_blocks_bit_exact(dtype):
    from paged_kv_cache_347_b200 import pagedattn as pa
    NB, Hkv, bs, D = 64, 8, 16, 128
    kc = _rand_bits((NB, Hkv, bs, D), dtype, 5)
    vc = _rand_bits((NB, Hkv, bs, D), dtype, 6)
    r = np.random.default_rng(0)
    blocks = r.permutation(NB)
    pairs = np.stack([blocks[:20], blocks[20:40]], 1).astype(np.int64)
    dk, dv = kc.cuda(), vc.cuda()
    pa.pa_copy_blocks(dk, dv, torch.from_numpy(pairs).cuda())
    cache_ref.copy_blocks(kc.view(BITS[dtype]), vc.view(BITS[dtype]), pairs.tolist())
    assert torch.equal(dk.cpu().view(BITS[dtype]), kc.view(BITS[dtype]))
    assert torch.equal(dv.cpu().view(BITS[dtype]), vc.view(BITS[dtype]))


def test_out_of_range_slots_and_pairs_are_flagged_and_skipped():
    from paged_kv_cache_347_b200 import pagedattn as pa
    pa.device_errors(clear=True)
    kc = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones(2, 1, 64, dtype=torch.bfloat16, device="cuda")
    pa.pa_reshape_and_cache(k, k, kc, vc, torch.tensor([64, 3], device="cuda"))
    assert pa.device_errors(clear=True) == ["slot"]
    assert kc.sum().item() == 64 and torch.all(kc[0, 0, 3] == 1)
    pa.pa_copy_blocks(kc, vc, torch.tensor([[0, 4]], device="cuda"))
    assert pa.device_errors(clear=True) == ["pair"]
    assert kc.sum().item() == 64


def test_long_context_prefill_cache_bit_exact():
    """The full-size 32k prefill (262k tokens) lands byte for byte."""
    wl = workloads.long_context(steps=1)
    sh = wl.shape
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    orc = OracleRun(sh)
    gpu = PagedKVRunner.for_shape(sh, 2048)
    st = next(iter(wl.steps))
    ref = orc.step(st, decode=False)
    acts = gpu.plan(st.ops)
    assert [int(x) for a in acts if a.kind == "write" for x in a.slots] == ref["slots"]
    gpu.upload(acts)
    gpu.execute(acts, st.k_new.cuda(), st.v_new.cuda(), None)
    torch.cuda.synchronize()
    assert torch.equal(gpu.k_cache.cpu().view(torch.int16), orc.k_cache.view(torch.int16))
    assert torch.equal(gpu.v_cache.cpu().view(torch.int16), orc.v_cache.view(torch.int16))


def test_beam_first_step_copies_twelve_blocks():
    """Step 1 of the beam workload: 3 copies per group of 4 beams, caches bit-exact."""
    wl = workloads.beam(steps=1)
    errs, gpu, orc = run_parity(wl, table_width=152, compare_cache=True)
    assert len(errs) == 1
    st = gpu.alloc.stats()
    assert st["used_blocks"] == 4 * (129 + 3) == orc.alloc.stats()["used_blocks"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_swap_blocks_device_host_round_trip_bit_exact(dtype):
    from paged_kv_cache_347_b200 import pagedattn as pa
    NB, NH, Hkv, bs, D = 48, 20, 4, 16, 128
    dk = _rand_bits((NB, Hkv, bs, D), dtype, 7).cuda()
    dv = _rand_bits((NB, Hkv, bs, D), dtype, 8).cuda()
    hk = torch.zeros((NH, Hkv, bs, D), dtype=DT[dtype]).pin_memory()
    hv = torch.zeros((NH, Hkv, bs, D), dtype=DT[dtype]).pin_memory()
    r = np.random.default_rng(3)
    out_pairs = np.stack([r.choice(NB, 12, replace=False), r.choice(NH, 12, replace=False)], 1)
    pa.pa_swap_blocks(hk, hv, dk, dv, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    b = BITS[dtype]
    ref_k = torch.zeros_like(hk).view(b); ref_v = torch.zeros_like(hv).view(b)
    cache_ref.copy_between(ref_k, ref_v, dk.cpu().view(b), dv.cpu().view(b), out_pairs.tolist())
    assert torch.equal(hk.view(b), ref_k) and torch.equal(hv.view(b), ref_v)
    # back into other device blocks, pairs given in pinned host memory
    in_pairs = np.stack([out_pairs[:, 1], r.choice(NB, 12, replace=False)], 1)
    dk2, dv2 = dk.clone(), dv.clone()
    pa.pa_swap_blocks(dk2, dv2, hk, hv, torch.from_numpy(in_pairs.copy()).pin_memory())
    torch.cuda.synchronize()
    ek, ev = dk.cpu().view(b).clone(), dv.cpu().view(b).clone()
    cache_ref.copy_between(ek, ev, hk.view(b), hv.view(b), in_pairs.tolist())
    assert torch.equal(dk2.cpu().view(b), ek) and torch.equal(dv2.cpu().view(b), ev)


def test_swap_blocks_rejects_pageable_host_memory():
    import ctypes
    from paged_kv_cache_347_b200 import pagedattn as pa
    dk = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    hk = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16)          # not pinned
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    rc = pa._lib.pa_swap_blocks(hk.data_ptr(), hk.data_ptr(), dk.data_ptr(), dk.data_ptr(),
                                pairs.data_ptr(), 1, 16 * 64 * 2, 4, 4, None)
    assert rc == -1 and b"page-locked" in pa._lib.pa_last_error()
    with pytest.raises(TypeError):
        pa.pa_swap_blocks(hk, hk, dk, dk, pairs)
