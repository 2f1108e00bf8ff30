"""Guard regions: every kernel writes only inside the buffers it is given.

compute-sanitizer is not available on the GPU pool, so stray stores are
looked for directly.  Each output buffer is carved out of a larger device
allocation whose first and last 4 KB hold a canary pattern (a NaN payload in
every dtype, so a stray read of it would also show in the results); after
the call the canaries must be bit-for-bit intact.  Inputs the call only reads
(q, caches, tables, lengths) must come back unchanged.  Needs a B200."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes before and after each buffer
CANARY = {2: 0x7FA5, 4: 0x7FA5A5A5}  # NaN in bf16, f16 and f32
BITS = {2: torch.int16, 4: torch.int32}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


class Guarded:
    """A tensor of `shape`/`dtype` in the middle of a canary-filled buffer
    (device, or pinned host memory when `pinned`)."""

    def __init__(self, shape, dtype, pinned=False):
        es = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape))
        self.g = GUARD // es
        kw = {"pin_memory": True} if pinned else {"device": "cuda"}
        self.raw = torch.full((self.g + self.n + self.g,), CANARY[es], dtype=BITS[es], **kw)
        self.t = self.raw[self.g:self.g + self.n].view(dtype).view(shape)
        self.canary = CANARY[es]

    def intact(self) -> bool:
        torch.cuda.synchronize()
        head, tail = self.raw[:self.g], self.raw[self.g + self.n:]
        return bool((head == self.canary).all()) and bool((tail == self.canary).all())


def _fill(gt: Guarded, src: torch.Tensor) -> Guarded:
    gt.t.copy_(src)
    return gt


def _paged_inputs(B, Hq, Hkv, D, bs, lens, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = max(1, max((L + bs - 1) // bs for L in lens))
    nb = sum((L + bs - 1) // bs for L in lens) + 3
    perm = torch.randperm(nb, generator=g, device="cuda").to(torch.int32)
    tab = torch.zeros(B, W, dtype=torch.int32, device="cuda")
    o = 0
    for b, L in enumerate(lens):
        n = (L + bs - 1) // bs
        tab[b, :n] = perm[o:o + n]
        o += n
    kc = torch.randn(nb, Hkv, bs, D, generator=g, device="cuda").to(dtype)
    vc = torch.randn(nb, Hkv, bs, D, generator=g, device="cuda").to(dtype)
    q = torch.randn(B, Hq, D, generator=g, device="cuda").to(dtype)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return q, kc, vc, tab, sl


def _snap(*ts):
    torch.cuda.synchronize()
    return [t.clone() for t in ts]


def _unchanged(before, after):
    for a, b in zip(before, after):
        es = a.element_size()
        assert torch.equal(a.reshape(-1).view(BITS.get(es, torch.int8)),
                           b.reshape(-1).view(BITS.get(es, torch.int8))), "an input was written"


@pytest.mark.parametrize("dtype,bs,D,G,lens", [
    (torch.bfloat16, 16, 128, 8, [1, 511, 512, 513, 3000, 0, 17]),  # tensor-core kernel, splits
    (torch.float16, 64, 64, 5, [64, 1100, 2]),
    (torch.float32, 4, 64, 2, [5, 9, 14, 700]),                    # CUDA-core kernel
    (torch.bfloat16, 4, 128, 4, [33, 1025]),
])
@pytest.mark.parametrize("variant,merge", [(0, 1), (0, 2), (3, 2)])
def test_decode_writes_only_out_and_its_workspace(dtype, bs, D, G, lens, variant, merge):
    from paged_kv_cache_347_b200 import pagedattn as pa
    if variant == 3 and dtype == torch.float32:
        pytest.skip("the tensor-core kernels take 16-bit caches")
    B, Hkv = len(lens), 2
    Hq = G * Hkv
    q, kc, vc, tab, sl = _paged_inputs(B, Hq, Hkv, D, bs, lens, dtype, 3)
    qg = _fill(Guarded(q.shape, dtype), q)
    kg = _fill(Guarded(kc.shape, dtype), kc)
    vg = _fill(Guarded(vc.shape, dtype), vc)
    out = Guarded((B, Hq, D), torch.float32)
    max_len = tab.shape[1] * bs
    need = pa.decode_workspace_size(B, Hq, D, max_len)
    ws = Guarded(((max(need, 16) + 15) // 16 * 4,), torch.float32)
    before = _snap(qg.t, kg.t, vg.t, tab, sl)
    pa.pa_decode(out.t, qg.t, kg.t, vg.t, tab, sl, 0.125, max_seq_len=max_len,
                 workspace=ws.t if need else None, variant=variant, merge=merge)
    assert out.intact() and ws.intact() and qg.intact() and kg.intact() and vg.intact()
    _unchanged(before, _snap(qg.t, kg.t, vg.t, tab, sl))
    assert torch.isfinite(out.t).all()
    assert not pa.device_errors()


def test_static_decode_writes_only_out():
    from paged_kv_cache_347_b200 import pagedattn as pa
    lens = [1, 600, 4096, 0]
    B, Hkv, G, D, bs = len(lens), 8, 4, 128, 16
    q, kc, vc, tab, sl = _paged_inputs(B, G * Hkv, Hkv, D, bs, lens, torch.bfloat16, 4)
    out = Guarded((B, G * Hkv, D), torch.float32)
    before = _snap(q, kc, vc, tab, sl)
    pa.pa_decode_static(out.t, q, kc, vc, tab, sl, 0.09)
    assert out.intact()
    _unchanged(before, _snap(q, kc, vc, tab, sl))
    assert not pa.device_errors()


@pytest.mark.parametrize("variant", [1, 2, 3, 4])
@pytest.mark.parametrize("G", [4, 7])
def test_prefill_writes_only_out(variant, G):
    from paged_kv_cache_347_b200 import pagedattn as pa
    Hkv, D, bs = 2, 128, 16
    lens = [300, 1000, 129, 40]
    chunks = [300, 77, 1, 0]   # a whole sequence, a chunk after context, one token, none
    B = len(lens)
    q_all, kc, vc, tab, sl = _paged_inputs(B, G * Hkv, Hkv, D, bs, lens, torch.bfloat16, 5)
    T = sum(chunks)
    g = torch.Generator(device="cuda").manual_seed(6)
    q = torch.randn(T, G * Hkv, D, generator=g, device="cuda").to(torch.bfloat16)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(chunks)]), dtype=torch.int32, device="cuda")
    out = Guarded((T, G * Hkv, D), torch.float32)
    before = _snap(q, kc, vc, tab, sl, cu)
    pa.pa_prefill(out.t, q, kc, vc, tab, sl, cu, 0.088, max_q_len=max(chunks),
                  max_seq_len=tab.shape[1] * bs, variant=variant)
    assert out.intact()
    _unchanged(before, _snap(q, kc, vc, tab, sl, cu))
    assert torch.isfinite(out.t).all()
    assert not pa.device_errors()


@pytest.mark.parametrize("variant", [2, 3, 4])
def test_prefill_output_16_byte_aligned(variant):
    """The tcgen05 kernels write a row with 32-byte stores when out is
    32-byte aligned and fall back to 16-byte ones when it is only 16-byte
    aligned: an out that starts 16 bytes into a buffer gets the same bits as
    an aligned one, and the 16 bytes before it and the tail stay untouched."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    G, Hkv, D, bs = 4, 2, 128, 16
    lens, chunks = [300, 1000, 129], [300, 77, 1]
    B = len(lens)
    _, kc, vc, tab, sl = _paged_inputs(B, G * Hkv, Hkv, D, bs, lens, torch.bfloat16, 9)
    T = sum(chunks)
    g = torch.Generator(device="cuda").manual_seed(10)
    q = torch.randn(T, G * Hkv, D, generator=g, device="cuda").to(torch.bfloat16)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(chunks)]), dtype=torch.int32, device="cuda")
    n = T * G * Hkv * D
    aligned = torch.empty(n, dtype=torch.float32, device="cuda")
    buf = torch.full((n + 8,), float("nan"), dtype=torch.float32, device="cuda")
    shifted = buf[4:4 + n]                      # 16 bytes past a 256-byte boundary
    assert shifted.data_ptr() % 32 == 16
    for o in (aligned, shifted):
        pa.pa_prefill(o.view(T, G * Hkv, D), q, kc, vc, tab, sl, cu, 0.088,
                      max_q_len=max(chunks), max_seq_len=tab.shape[1] * bs, variant=variant)
    torch.cuda.synchronize()
    assert torch.equal(aligned.view(torch.int32), shifted.view(torch.int32))
    assert torch.isnan(buf[:4]).all() and torch.isnan(buf[4 + n:]).all()
    assert not pa.device_errors()


@pytest.mark.parametrize("dtype,bs,D", [(torch.bfloat16, 16, 128), (torch.float32, 4, 64),
                                        (torch.float16, 64, 64)])
def test_append_writes_only_its_slots(dtype, bs, D):
    from paged_kv_cache_347_b200 import pagedattn as pa
    NB, Hkv, N = 40, 3, 50
    r = np.random.default_rng(7)
    slots = r.choice(NB * bs, size=N, replace=False).astype(np.int64)
    slots[:2] = [0, NB * bs - 1]            # the first and the last slot of the pool
    slots[5] = -1                           # skipped
    g = torch.Generator(device="cuda").manual_seed(8)
    k = torch.randn(N, Hkv, D, generator=g, device="cuda").to(dtype)
    v = torch.randn(N, Hkv, D, generator=g, device="cuda").to(dtype)
    kc = _fill(Guarded((NB, Hkv, bs, D), dtype), torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(dtype))
    vc = _fill(Guarded((NB, Hkv, bs, D), dtype), torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(dtype))
    kb, vb = _snap(kc.t, vc.t)
    pa.pa_reshape_and_cache(k, v, kc.t, vc.t, torch.from_numpy(slots).cuda())
    assert kc.intact() and vc.intact()
    # every slot not in the mapping keeps its bits
    written = torch.zeros(NB * bs, dtype=torch.bool)
    written[torch.from_numpy(slots[slots >= 0])] = True
    keep = (~written).view(NB, 1, bs, 1).expand(NB, Hkv, bs, D).reshape(-1)
    es = kb.element_size()
    for before, now in ((kb, kc.t), (vb, vc.t)):
        a = before.reshape(-1).view(BITS[es]).cpu()[keep]
        b = now.reshape(-1).view(BITS[es]).cpu()[keep]
        assert torch.equal(a, b)
    assert not pa.device_errors()


def test_copy_blocks_writes_only_destination_blocks():
    from paged_kv_cache_347_b200 import pagedattn as pa
    NB, Hkv, bs, D = 24, 8, 16, 128
    g = torch.Generator(device="cuda").manual_seed(9)
    kc = _fill(Guarded((NB, Hkv, bs, D), torch.bfloat16),
               torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(torch.bfloat16))
    vc = _fill(Guarded((NB, Hkv, bs, D), torch.bfloat16),
               torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(torch.bfloat16))
    pairs = torch.tensor([[NB - 2, NB - 1], [3, 0], [5, 6]], dtype=torch.int64)  # the pool's ends as destinations
    kb, vb = _snap(kc.t, vc.t)
    pa.pa_copy_blocks(kc.t, vc.t, pairs.cuda())
    assert kc.intact() and vc.intact()
    dst = {0, NB - 1, 6}
    for before, now in ((kb, kc.t), (vb, vc.t)):
        for blk in range(NB):
            if blk not in dst:
                assert torch.equal(before[blk].view(torch.int16), now[blk].view(torch.int16))
    assert not pa.device_errors()


def test_swap_writes_only_destination_blocks_on_either_side():
    from paged_kv_cache_347_b200 import pagedattn as pa
    NB, NH, Hkv, bs, D = 16, 12, 2, 16, 64
    g = torch.Generator(device="cuda").manual_seed(10)
    dk = _fill(Guarded((NB, Hkv, bs, D), torch.bfloat16),
               torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(torch.bfloat16))
    dv = _fill(Guarded((NB, Hkv, bs, D), torch.bfloat16),
               torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(torch.bfloat16))
    hk = Guarded((NH, Hkv, bs, D), torch.bfloat16, pinned=True)
    hv = Guarded((NH, Hkv, bs, D), torch.bfloat16, pinned=True)
    hk.t.zero_()
    hv.t.zero_()
    out_pairs = torch.tensor([[0, NH - 1], [NB - 1, 0], [3, 4]], dtype=torch.int64, device="cuda")
    pa.pa_swap_blocks(hk.t, hv.t, dk.t, dv.t, out_pairs)      # device -> host
    assert hk.intact() and hv.intact() and dk.intact() and dv.intact()
    for src, dst in ((0, NH - 1), (NB - 1, 0), (3, 4)):
        assert torch.equal(hk.t[dst].view(torch.int16), dk.t[src].cpu().view(torch.int16))
    untouched = [b for b in range(NH) if b not in (NH - 1, 0, 4)]
    assert (hk.t[untouched].view(torch.int16) == 0).all()
    kb = _snap(dk.t)[0]
    in_pairs = torch.tensor([[NH - 1, 2], [0, NB - 1]], dtype=torch.int64, device="cuda")
    pa.pa_swap_blocks(dk.t, dv.t, hk.t, hv.t, in_pairs)       # host -> device
    assert hk.intact() and dk.intact() and dv.intact()
    for blk in range(NB):
        if blk not in (2, NB - 1):
            assert torch.equal(kb[blk].view(torch.int16), dk.t[blk].view(torch.int16))
    assert torch.equal(dk.t[2].view(torch.int16), kb[0].view(torch.int16))
    assert not pa.device_errors()
