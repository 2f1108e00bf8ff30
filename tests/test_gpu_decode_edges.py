"""Decode edge cases against the fp64 oracle (needs a B200).

Paging must not change the attention result (paweldubiel.com
"PagedAttention", "Text order is not a memory address") on any input the
method can meet, so these cases feed what the workload tests never do:

* slots past each sequence's length in its last block, blocks no table
  names, and table entries past a sequence's last block hold NaN, +Inf or
  -Inf -- the oracle never reads them and neither may the kernels;
* logits of magnitude ~1e3 (queries scaled up), where the softmax is nearly
  one-hot and any missing max subtraction overflows;
* a scale of 0 (the plain mean of the values) and negative scales (the order
  of the softmax reversed);
* lengths on both sides of the 16-token MMA tile, the 32-token stage and the
  512-token split.

Every decode kernel runs every case: variant 1 (CUDA cores, every dtype and
block size), variant 2 (tensor cores, 16-bit caches; blocks of 4 rows staged
by cp.async, larger ones by TMA) and variant 3 (tensor cores, one KV head per
warp).
Tolerances: max-abs 1e-5 for fp32 caches, 3e-3 for bf16 / f16; at logits of
~1e3 the fp32 caches add the bound that fp32 rounding of the logits itself
puts on the output (``_fp32_logit_tolerance``)."""
import numpy as np
import pytest
import torch

from parity import TOL
import workloads

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
LENS = [0, 1, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1023, 1025, 1537]


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_347_b200 import pagedattn
    pagedattn.device_errors(clear=True)
    yield pagedattn
    assert pagedattn.device_errors(clear=True) == []


def _case(seed, lens, Hq, Hkv, D, bs, dtype, q_scale=1.0, fill=None):
    """Host caches, tables and queries.  Every sequence's blocks are drawn from
    a seeded permutation of the pool; with ``fill``, everything the attention
    must not read is set to that value: the slots past L in each last block,
    the blocks that no table names, and one spare block that the table
    entries past each sequence's last block point to."""
    nblk = [-(-L // bs) for L in lens]
    W = max(max(nblk), 1) + 2
    NB = sum(nblk) + 8
    perm = workloads.permutation(seed, NB)
    kc = workloads.normal(seed, (1,), (NB, Hkv, bs, D), dtype)
    vc = workloads.normal(seed, (2,), (NB, Hkv, bs, D), dtype)
    q = workloads.normal(seed, (3,), (len(lens), Hq, D), "f32") * q_scale
    q = q.to(TORCH_DT[dtype])
    spare = int(perm[-1])
    tables = np.full((len(lens), W), spare, np.int32)
    used = set()
    o = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[o:o + n]
        used.update(int(b) for b in perm[o:o + n])
        o += n
    if fill is not None:
        for b in range(NB):
            if b not in used:
                kc[b] = fill
                vc[b] = fill
        for s, L in enumerate(lens):
            if L % bs:
                last = int(tables[s, (L - 1) // bs])
                kc[last, :, L % bs:, :] = fill
                vc[last, :, L % bs:, :] = fill
    return q, kc, vc, tables, np.asarray(lens, np.int32)


def _run(pa, q, kc, vc, tables, lens, scale, variant, partition=0, max_seq_len=None):
    dev = [t.cuda() for t in (q, kc, vc)]
    tab = torch.from_numpy(tables).cuda()
    sl = torch.from_numpy(lens).cuda()
    out = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_decode(out, dev[0], dev[1], dev[2], tab, sl, scale, partition_size=partition,
                 variant=variant, max_seq_len=max_seq_len)
    torch.cuda.synchronize()
    return out.double().cpu().numpy()


def _check(got, exp, dtype, what):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = float(np.abs(got - exp).max())
    assert err <= TOL[dtype], f"{what}: max-abs {err}"
    return err


KERNELS = [(1, "f32", 4), (1, "f32", 16), (1, "bf16", 4), (1, "f16", 16),
           (2, "bf16", 4), (2, "f16", 4), (2, "bf16", 8), (2, "bf16", 16), (2, "f16", 32),
           (2, "bf16", 64), (3, "bf16", 4), (3, "f16", 8), (3, "bf16", 16), (3, "f16", 32),
           (3, "bf16", 64)]


@pytest.mark.parametrize("fill", [float("nan"), float("inf"), float("-inf")])
@pytest.mark.parametrize("variant,dtype,bs", KERNELS)
def test_poisoned_slots_are_never_read(pa, variant, dtype, bs, fill):
    from oracle import attn
    Hq, Hkv, D = 8, 2, 128
    q, kc, vc, tables, lens = _case(21, LENS, Hq, Hkv, D, bs, dtype, fill=fill)
    scale = D ** -0.5
    exp = attn.paged_decode(q, kc, vc, tables, lens, scale)
    got = _run(pa, q, kc, vc, tables, lens, scale, variant)
    _check(got, exp, dtype, f"variant {variant} {dtype} bs {bs} fill {fill}")
    # an empty sequence still gives zeros next to poisoned neighbours
    assert np.all(got[0] == 0.0)


def _fp32_logit_tolerance(q, kc, vc, tables, lens, scale, G):
    """Per (sequence, head) bound on what rounding the logits to fp32 does to
    the output, for fp32 caches.  A perturbation d_t of the logits moves the
    output by sum_t w_t (d_t - sum_u w_u d_u)(v_t - out), so |d_t| <= eps
    bounds it by 2 eps sum_t w_t |v_t - out|.  The kernels form each logit as
    a sum of D products with at most 2 log2(D) + 4 roundings on any path (FMA
    chains and a shuffle tree), then scale it, shift it by the running maximum
    and exponentiate; eps = 16 u max_t sum_d |scale q_d k_td| with u = 2^-24
    covers all of it.  At |logits| ~ 1e3 that is ~1e-3, against rounding
    effects of ~1e-4 in a float32 emulation of these inputs: the 1e-5 bound
    stated for N(0, 1) data cannot hold there for any fp32 kernel (half an
    ulp of 1000.0 in fp32 is already 3e-5)."""
    from oracle import attn
    qd, kd, vd = (attn.decode_storage(t) for t in (q, kc, vc))
    B, Hq, D = qd.shape
    tol = np.zeros((B, Hq))
    for s, L in enumerate(lens):
        for h in range(Hq):
            if L == 0:
                continue
            K = attn.gather_logical(kd, tables[s], int(L), h // G)
            V = attn.gather_logical(vd, tables[s], int(L), h // G)
            x = scale * (K @ qd[s, h])
            w = np.exp(x - x.max())
            w /= w.sum()
            out = w @ V
            eps = 16 * 2.0 ** -24 * float((np.abs(K) @ np.abs(qd[s, h])).max()) * abs(scale)
            tol[s, h] = 2 * eps * float((w @ np.abs(V - out)).max())
    return tol


@pytest.mark.parametrize("variant,dtype,bs", KERNELS)
@pytest.mark.parametrize("G", [1, 4, 8])
def test_logits_of_magnitude_one_thousand(pa, variant, dtype, bs, G):
    """Queries scaled so that scale * q.k reaches about +-1e3: the softmax is
    close to one-hot, exp of an unshifted logit would overflow fp32, and the
    online rescale sees running maxima jump by hundreds.  16-bit caches keep
    the 3e-3 bound; fp32 caches get 1e-5 plus the fp32 logit-rounding bound
    of ``_fp32_logit_tolerance``."""
    from oracle import attn
    Hkv, D = 2, 128
    lens = [1, 17, 33, 513, 1100]
    q, kc, vc, tables, lens = _case(22, lens, G * Hkv, Hkv, D, bs, dtype, q_scale=300.0,
                                    fill=float("nan"))
    scale = D ** -0.5
    qd = attn.decode_storage(q)
    kd = attn.decode_storage(kc)
    # the logits really are that large
    big = max(float(np.abs(scale * attn.gather_logical(kd, tables[s], int(L), 0) @ qd[s, 0]).max())
              for s, L in enumerate(lens))
    assert big > 500.0, big
    exp = attn.paged_decode(q, kc, vc, tables, lens, scale)
    got = _run(pa, q, kc, vc, tables, lens, scale, variant)
    assert np.isfinite(got).all()
    err = np.abs(got - exp).max(axis=2)
    tol = TOL[dtype]
    if dtype == "f32":
        tol = tol + _fp32_logit_tolerance(q, kc, vc, tables, lens, scale, G)
    assert np.all(err <= tol), (float(err.max()), np.argwhere(err > tol)[:4].tolist())


@pytest.mark.parametrize("variant,dtype,bs", KERNELS)
@pytest.mark.parametrize("scale", [0.0, -0.05, -1.0 / 128 ** 0.5])
def test_zero_and_negative_scale(pa, variant, dtype, bs, scale):
    from oracle import attn
    Hq, Hkv, D = 8, 2, 128
    lens = [1, 16, 33, 600, 1025]
    q, kc, vc, tables, lens = _case(23, lens, Hq, Hkv, D, bs, dtype, fill=float("nan"))
    exp = attn.paged_decode(q, kc, vc, tables, lens, scale)
    got = _run(pa, q, kc, vc, tables, lens, scale, variant)
    _check(got, exp, dtype, f"variant {variant} {dtype} bs {bs} scale {scale}")
    if scale == 0.0:
        # every weight is 1: the output is the mean of the sequence's values
        vd = attn.decode_storage(vc)
        for s, L in enumerate(lens):
            rows = attn.gather_logical(vd, tables[s], int(L), 0)
            assert np.abs(got[s, 0] - rows.mean(axis=0)).max() <= TOL[dtype]


@pytest.mark.parametrize("variant,dtype,bs", [(1, "f32", 16), (1, "bf16", 8), (2, "bf16", 16),
                                              (2, "f16", 8), (3, "bf16", 16), (3, "f16", 4),
                                              (3, "bf16", 32)])
@pytest.mark.parametrize("partition", [64, 512, 1024])
def test_lengths_around_tiles_stages_and_splits(pa, variant, dtype, bs, partition):
    """Every length from 1 to 70 (tiles of 16, stages of 32 and 64 tokens)
    and the lengths on both sides of the split edges, one batch per split
    length."""
    from oracle import attn
    Hq, Hkv, D = 16, 4, 64
    lens = list(range(0, 71)) + [partition + d for d in (-1, 0, 1)] + \
           [2 * partition + d for d in (-1, 0, 1)] + [3 * partition - 17]
    q, kc, vc, tables, lens = _case(24 + partition, lens, Hq, Hkv, D, bs, dtype,
                                    fill=float("inf"))
    scale = D ** -0.5
    exp = attn.paged_decode(q, kc, vc, tables, lens, scale)
    got = _run(pa, q, kc, vc, tables, lens, scale, variant, partition=partition)
    _check(got, exp, dtype, f"variant {variant} {dtype} bs {bs} split {partition}")


# ---------------------------------------------------------------- split merges
@pytest.mark.parametrize("variant,dtype,bs", [(1, "f32", 16), (2, "bf16", 16), (3, "f16", 8)])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("max_splits", [2, 8, 9, 16, 17, 32, 33, 64, 65, 130])
def test_every_form_of_the_split_reduce(pa, variant, dtype, bs, D, max_splits):
    """The reduce gives a (sequence, query head) 1, 2 or 4 warps, or a whole
    CTA, from the longest sequence's split count and the rows a warp-wide
    load covers (one at D 128, two at D 64); its lanes batch 8 rows at a
    time.  64-token splits and a longest sequence of exactly ``max_splits``
    splits put every form and both sides of each boundary under test, next
    to shorter sequences (one split, none, a split edge) in the same batch."""
    from oracle import attn
    Hq, Hkv = 8, 2
    part = 64
    top = max_splits * part
    lens = [0, 1, part - 1, part, part + 1, max(1, top - part - 5), top - 3, top]
    q, kc, vc, tables, lens = _case(31 + max_splits, lens, Hq, Hkv, D, bs, dtype,
                                    fill=float("nan"))
    scale = D ** -0.5
    exp = attn.paged_decode(q, kc, vc, tables, lens, scale)
    # the bound is the longest length, so the launch has exactly max_splits
    got = _run(pa, q, kc, vc, tables, lens, scale, variant, partition=part,
               max_seq_len=int(lens.max()))
    _check(got, exp, dtype, f"variant {variant} D {D} splits {max_splits}")
    assert np.all(got[0] == 0.0)


@pytest.mark.parametrize("variant,dtype,bs", [(1, "f32", 16), (1, "bf16", 4), (2, "bf16", 16),
                                              (2, "f16", 8), (3, "bf16", 16), (3, "f16", 8)])
@pytest.mark.parametrize("partition", [64, 512])
def test_in_kernel_merge_and_reduce_kernel_agree_with_the_oracle(pa, variant, dtype, bs,
                                                                  partition):
    """Both ways of combining the split partials -- the reduce kernel (merge
    1) and the last CTA of each (sequence, KV head) inside the main kernel
    (merge 2) -- on a workspace full of old bytes (the tickets are never
    cleared), two calls in a row."""
    from oracle import attn
    Hq, Hkv, D = 16, 4, 128
    lens = [0, 1, 63, 64, 65, 700, 1025, 2 * partition + 5, 9 * partition]
    q, kc, vc, tables, lens = _case(31, lens, Hq, Hkv, D, bs, dtype, fill=float("nan"))
    scale = D ** -0.5
    exp = attn.paged_decode(q, kc, vc, tables, lens, scale)
    dev = [t.cuda() for t in (q, kc, vc)]
    tab, sl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    need = pa.decode_workspace_size(len(lens), Hq, D, tables.shape[1] * bs, partition)
    ws = torch.randint(0, 256, (need,), dtype=torch.uint8, device="cuda")
    for merge in (1, 2, 2, 1, 2):
        out = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device="cuda")
        pa.pa_decode(out, dev[0], dev[1], dev[2], tab, sl, scale, workspace=ws,
                     partition_size=partition, variant=variant, merge=merge)
        torch.cuda.synchronize()
        _check(out.double().cpu().numpy(), exp, dtype, f"merge {merge}")


def test_in_kernel_merge_replays_from_a_cuda_graph(pa):
    """A graph replays the same call (the same ticket tag) with new inputs:
    each replay finds the tickets its previous run reset, and matches the
    oracle."""
    from oracle import attn
    Hq, Hkv, D, bs = 32, 8, 128, 16
    lens = [1500, 2049, 33, 4000]
    q, kc, vc, tables, lens = _case(32, lens, Hq, Hkv, D, bs, "bf16")
    scale = D ** -0.5
    dq, dk, dv = (t.cuda() for t in (q, kc, vc))
    tab, sl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    need = pa.decode_workspace_size(len(lens), Hq, D, tables.shape[1] * bs, 512)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty(tuple(q.shape), dtype=torch.float32, device="cuda")
    run = lambda: pa.pa_decode(out, dq, dk, dv, tab, sl, scale, workspace=ws, partition_size=512,
                               merge=2)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run()
    for k in range(3):
        qk = workloads.normal(40 + k, (3,), tuple(q.shape), "f32").to(q.dtype)
        dq.copy_(qk)
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        exp = attn.paged_decode(qk, kc, vc, tables, lens, scale)
        _check(out.double().cpu().numpy(), exp, "bf16", f"replay {k}")
    del g


@pytest.mark.parametrize("heads_per_cta", [1, 2, 4])
@pytest.mark.parametrize("G,Hkv", [(1, 8), (4, 8), (8, 4), (3, 4)])
def test_heads_per_cta(pa, heads_per_cta, G, Hkv):
    """Variant 3 with 1, 2 or 4 KV heads per CTA (one per warp) on every
    GQA group size the tiles hold, against the oracle."""
    from oracle import attn
    D, bs = 128, 16
    lens = [0, 1, 17, 511, 513, 1600]
    q, kc, vc, tables, lens = _case(33, lens, G * Hkv, Hkv, D, bs, "bf16", fill=float("nan"))
    scale = D ** -0.5
    exp = attn.paged_decode(q, kc, vc, tables, lens, scale)
    dev = [t.cuda() for t in (q, kc, vc)]
    out = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_decode(out, dev[0], dev[1], dev[2], torch.from_numpy(tables).cuda(),
                 torch.from_numpy(lens).cuda(), scale, variant=3, heads_per_cta=heads_per_cta)
    torch.cuda.synchronize()
    _check(out.double().cpu().numpy(), exp, "bf16", f"{heads_per_cta} heads per CTA")


@pytest.mark.parametrize("variant", [1, 2, 3])
def test_dispatch_order_changes_nothing_but_the_schedule(pa, variant):
    """The grid taking the sequences longest first (seq_order) gives outputs
    bit-identical to the batch order: each (sequence, head) is computed by the
    same CTA code over the same tokens.  An entry outside the batch skips its
    row and raises the length error bit."""
    Hq, Hkv, D, bs = 16, 4, 128, 16
    lens = [700, 1, 3000, 0, 64, 1500, 100]   # the last row fits one split
    q, kc, vc, tables, lens = _case(34, lens, Hq, Hkv, D, bs, "bf16")
    dev = [t.cuda() for t in (q, kc, vc)]
    tab, sl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    outs = []
    for order in (None, pa.decode_order(lens)):
        out = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device="cuda")
        pa.pa_decode(out, dev[0], dev[1], dev[2], tab, sl, D ** -0.5, variant=variant,
                     seq_order=None if order is None else torch.from_numpy(order).cuda())
        torch.cuda.synchronize()
        outs.append(out.cpu())
    assert torch.equal(outs[0], outs[1])
    bad = torch.tensor([2, 0, 1, 3, 4, 5, 99], dtype=torch.int32, device="cuda")
    out = torch.zeros(tuple(q.shape), dtype=torch.float32, device="cuda")
    pa.device_errors(clear=True)
    pa.pa_decode(out, dev[0], dev[1], dev[2], tab, sl, D ** -0.5, variant=variant,
                 seq_order=bad)
    assert pa.device_errors(clear=True) == ["seqlen"]
    torch.cuda.synchronize()
    assert torch.all(out[6] == 0)          # the row no grid row named
    assert torch.equal(out[:6].cpu(), outs[0][:6])
