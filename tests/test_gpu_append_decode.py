"""pa_append_decode: a decode step's one-token appends written by the decode
kernel itself, against the separate append + decode and the fp64 oracle
(needs a B200).  The caches must come out bit for bit as the separate append
leaves them; the outputs match the oracle within the path's tolerance."""
import numpy as np
import pytest
import torch

from parity import TOL
import workloads

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_347_b200 import pagedattn
    pagedattn.device_errors(clear=True)
    yield pagedattn
    assert pagedattn.device_errors(clear=True) == []


def _step(seed, lens, Hq, Hkv, D, bs, dtype):
    """Caches holding L_s - 1 tokens of each sequence, the new token's K/V and
    its slot (position L_s - 1), queries, tables."""
    nblk = [-(-L // bs) for L in lens]
    W = max(nblk) + 1
    NB = sum(nblk) + 5
    perm = workloads.permutation(seed, NB)
    tables = np.zeros((len(lens), W), np.int32)
    o = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[o:o + n]
        o += n
    kc = workloads.normal(seed, (1,), (NB, Hkv, bs, D), dtype)
    vc = workloads.normal(seed, (2,), (NB, Hkv, bs, D), dtype)
    slots = np.array([int(tables[s, (L - 1) // bs]) * bs + (L - 1) % bs if L > 0 else -1
                      for s, L in enumerate(lens)], np.int64)
    for s, L in enumerate(lens):   # the new position holds stale bytes before the step
        if L > 0:
            kc[slots[s] // bs, :, slots[s] % bs] = 7.0
            vc[slots[s] // bs, :, slots[s] % bs] = -7.0
    k_new = workloads.normal(seed, (3,), (len(lens), Hkv, D), dtype)
    v_new = workloads.normal(seed, (4,), (len(lens), Hkv, D), dtype)
    q = workloads.normal(seed, (5,), (len(lens), Hq, D), dtype)
    return q, kc, vc, k_new, v_new, slots, tables, np.asarray(lens, np.int32)


CASES = [(1, "f32", 4), (1, "bf16", 16), (2, "bf16", 16), (2, "f16", 4), (2, "bf16", 32),
         (3, "bf16", 16), (3, "f16", 8)]


@pytest.mark.parametrize("variant,dtype,bs", CASES)
@pytest.mark.parametrize("partition", [64, 512])
def test_fused_append_equals_the_separate_append(pa, variant, dtype, bs, partition):
    from oracle import attn, cache_ref
    Hq, Hkv, D = 16, 4, 128
    lens = [1, 2, 17, 64, 65, 600, 1500, 0, 33]
    q, kc, vc, kn, vn, slots, tables, lens = _step(41, lens, Hq, Hkv, D, bs, dtype)
    scale = D ** -0.5
    dev = lambda t: t.cuda()
    tab, sl, sm = (torch.from_numpy(x).cuda() for x in (tables, lens, slots))
    # separate: pa_reshape_and_cache, then pa_decode
    kc1, vc1 = dev(kc), dev(vc)
    live = torch.from_numpy(slots >= 0)
    pa.pa_reshape_and_cache(dev(kn), dev(vn), kc1, vc1, sm)
    out1 = torch.empty(tuple(q.shape), dtype=torch.float32, device="cuda")
    pa.pa_decode(out1, dev(q), kc1, vc1, tab, sl, scale, partition_size=partition,
                 variant=variant)
    # fused
    kc2, vc2 = dev(kc), dev(vc)
    out2 = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_append_decode(out2, dev(q), dev(kn), dev(vn), sm, kc2, vc2, tab, sl, scale,
                        partition_size=partition, variant=variant)
    torch.cuda.synchronize()
    bits = torch.int32 if dtype == "f32" else torch.int16
    assert torch.equal(kc1.view(bits), kc2.view(bits)) and torch.equal(vc1.view(bits), vc2.view(bits))
    # and against the oracle: the append on host caches, then the fp64 decode
    kh, vh = kc.clone(), vc.clone()
    cache_ref.reshape_and_cache(kn, vn, kh, vh, slots)
    exp = attn.paged_decode(q, kh, vh, tables, lens, scale)
    got = out2.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert float(np.abs(got - exp).max()) <= TOL[dtype]
    assert torch.equal(kc2.cpu().view(bits), kh.view(bits))
    # the same CTAs compute the same sums either way
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("variant", [1, 2, 3])
def test_a_slot_that_is_not_the_new_position_is_refused(pa, variant):
    """A slot other than position L - 1's (which another CTA could be
    reading) is not written and sets the slot error bit; a negative slot
    writes nothing and is no error."""
    Hq, Hkv, D, bs = 8, 2, 128, 16
    lens = [40, 100, 7]
    q, kc, vc, kn, vn, slots, tables, lens = _step(42, lens, Hq, Hkv, D, bs, "bf16")
    bad = slots.copy()
    bad[1] = int(tables[1, 0]) * bs + 3      # a slot in the sequence's first block
    bad[2] = -1
    kc_d, vc_d = kc.cuda(), vc.cuda()
    out = torch.empty(tuple(q.shape), dtype=torch.float32, device="cuda")
    pa.device_errors(clear=True)
    pa.pa_append_decode(out, q.cuda(), kn.cuda(), vn.cuda(), torch.from_numpy(bad).cuda(),
                        kc_d, vc_d, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                        D ** -0.5, variant=variant)
    assert pa.device_errors(clear=True) == ["slot"]
    kc_h = kc_d.cpu()
    # sequence 0 appended; sequences 1 and 2 left their caches untouched
    assert torch.equal(kc_h[slots[0] // bs, :, slots[0] % bs].view(torch.int16),
                       kn[0].view(torch.int16))
    for s in (1, 2):
        assert torch.equal(kc_h[slots[s] // bs, :, slots[s] % bs].view(torch.int16),
                           kc[slots[s] // bs, :, slots[s] % bs].view(torch.int16))
        assert torch.equal(kc_h[bad[1] // bs].view(torch.int16), kc[bad[1] // bs].view(torch.int16))
