"""Parity of the CUDA decode path against the fp64 oracle (needs a B200).

Tolerances are the ones the path is built to: max-abs 1e-5 on the fp32 output
for fp32 caches, 3e-3 for bf16/f16 caches.  Each case runs the same seeded
events through oracle/run.py and paged_kv_cache_347_b200.runner, and checks
slots and copy pairs bit for bit on the way."""
import math

import numpy as np
import pytest
import torch

from conftest import golden
from parity import TOL, run_parity, sample_pairs
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_347_b200 import pagedattn as pa
    pa.device_errors(clear=True)
    yield pa
    assert pa.device_errors(clear=True) == []


def _pa():
    from paged_kv_cache_347_b200 import pagedattn as pa
    return pa


# ---------------------------------------------------------------- page examples
@pytest.mark.parametrize("dtype,bs,variant", [(torch.float32, 4, 0), (torch.bfloat16, 8, 2),
                                              (torch.float16, 16, 2), (torch.bfloat16, 4, 1)])
def test_scalar_example_on_gpu(dtype, bs, variant):
    """Keys 0, query 1, values 1..5 -> exactly 3 in both layouts; 1..L -> (L+1)/2."""
    pa = _pa()
    g = golden("scalar_example.json")
    D = 64
    for L in range(1, 17):
        layouts = [list(range(8))[: -(-L // bs)], [7, 2, 5, 0, 3, 6, 1, 4][: -(-L // bs)]]
        if L == g["length"] and bs == g["block_size"]:
            layouts = [[4, 1], [0, 1]]
        for layout in layouts:
            kc = torch.zeros(8, 1, bs, D, dtype=dtype, device="cuda")
            vc = torch.zeros_like(kc)
            for t in range(L):
                vc[layout[t // bs], 0, t % bs, 0] = float(g["values"][t] if t < 5 else t + 1)
            q = torch.zeros(1, 1, D, dtype=dtype, device="cuda")
            q[0, 0, 0] = g["query"]
            bt = torch.tensor([layout + [0] * (8 - len(layout))], dtype=torch.int32, device="cuda")
            sl = torch.tensor([L], dtype=torch.int32, device="cuda")
            out = torch.empty(1, 1, D, dtype=torch.float32, device="cuda")
            pa.pa_decode(out, q, kc, vc, bt, sl, 0.125, variant=variant)
            o = out.cpu()
            assert o[0, 0, 0].item() == (L + 1) / 2
            if L == g["length"]:
                assert o[0, 0, 0].item() == g["expected"]
            assert torch.all(o[0, 0, 1:] == 0)


# ---------------------------------------------------------------- workloads
def test_tiny_workload():
    errs, gpu, orc = run_parity(workloads.tiny(), table_width=4, compare_cache=True)
    assert len(errs) == 2 and max(errs) <= TOL["f32"], errs
    assert gpu.alloc.stats()["used_blocks"] == 9


@pytest.mark.parametrize("variant", [1, 2, 3])
def test_llama_shaped_reduced(variant):
    wl = workloads.llama(batch=6, lo=1, hi=700, steps=3, num_blocks=512)
    errs, _, _ = run_parity(wl, table_width=48, variant=variant, compare_cache=True)
    assert max(errs) <= TOL["bf16"], errs


def test_llama_shaped_full_sampled():
    wl = workloads.llama(steps=2)
    errs, _, _ = run_parity(wl, table_width=257, sample=48)
    assert max(errs) <= TOL["bf16"], errs


def test_llama_shaped_with_chosen_partition():
    """The runner's per-step split length (pa_decode_partition_for, asking the
    device for its slot count): the Llama-8B-shaped batch leaves 512-token
    CTAs part-way into a second wave on a B200, so a longer split is chosen;
    sampled outputs still match the oracle."""
    pa = _pa()
    wl = workloads.llama(steps=2)
    errs, gpu, _ = run_parity(wl, table_width=257, sample=48, partition_size=-1)
    assert max(errs) <= TOL["bf16"], errs
    lens = np.random.default_rng(1).integers(512, 4096, size=32, endpoint=True)
    p = pa.decode_partition_for(lens, 8, 128, 16, torch.bfloat16)
    assert p in (512, 1024)
    # the long-context batch is many waves deep at 512 and keeps it
    assert pa.decode_partition_for([32768] * 8, 8, 128, 16, torch.bfloat16) == 512


@pytest.mark.parametrize("partition", [64, 512, 1024])
def test_long_context_reduced(partition):
    wl = workloads.long_context(batch=2, seq_len=4096 + 37, steps=2, num_blocks=1024)
    errs, _, _ = run_parity(wl, table_width=260, partition_size=partition)
    assert max(errs) <= TOL["bf16"], errs


def test_long_context_full_sampled():
    wl = workloads.long_context(steps=1)
    errs, _, _ = run_parity(wl, table_width=2048, sample=24, check_slots=True)
    assert max(errs) <= TOL["bf16"], errs


def test_beam_cow_and_decode():
    """Step 1 makes 12 copy-on-write pairs; step 15 appends position 2064, so
    every beam opens its second private block; the caches stay bit-exact
    after every step and every output matches (mbrenndoerfer.com "Paged
    Attention > Summary", bullet 4: beams share the prompt's blocks)."""
    wl = workloads.beam(steps=18)
    errs, gpu, orc = run_parity(wl, table_width=152, compare_cache=True)
    assert len(errs) == 18 and max(errs) <= TOL["f16"], errs
    st = gpu.alloc.stats()
    # 4 prompts x (128 shared blocks + 4 beams x 2 private blocks)
    assert st["used_blocks"] == 4 * (128 + 4 * 2) == orc.alloc.stats()["used_blocks"]
    assert st["shared_blocks"] == 4 * 128


@pytest.mark.parametrize("bs", [8, 16, 32, 64])
def test_mix_reduced(bs):
    wl = workloads.mix(block_size=bs, steps=4, batch=24, hi=1500, pool_slots=65536)
    errs, _, _ = run_parity(wl, table_width=1600 // bs + 2)
    assert max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_mix_full_sampled(bs):
    wl = workloads.mix(block_size=bs, steps=2)
    errs, _, _ = run_parity(wl, table_width=8192 // bs + 8, sample=32)
    assert max(errs) <= TOL["bf16"], errs


# ---------------------------------------------------------------- properties
def test_placement_permutation_gives_bit_identical_outputs():
    outs = []
    for perm in (False, True):
        wl = workloads.custom("perm", [5, 9, 14, 100, 700], 8, 2, 128, "bf16", 16, 256, seed=11,
                              steps=1, permute=perm)
        errs, gpu, _ = run_parity(wl, table_width=48)
        assert max(errs) <= TOL["bf16"]
        outs.append(gpu)
    # rerun both to collect the raw outputs
    res = []
    for perm in (False, True):
        wl = workloads.custom("perm", [5, 9, 14, 100, 700], 8, 2, 128, "bf16", 16, 256, seed=11,
                              steps=1, permute=perm)
        from paged_kv_cache_347_b200.runner import PagedKVRunner
        r = PagedKVRunner.for_shape(wl.shape, 48)
        out = None
        for st in wl.steps:
            o = r.run(st)
            out = o if o is not None else out
        res.append(out.cpu())
    assert torch.equal(res[0], res[1])


@pytest.mark.parametrize("dtype,G,D,bs", [("bf16", 1, 128, 16), ("bf16", 3, 64, 8),
                                          ("f16", 8, 64, 32), ("f32", 4, 128, 16),
                                          ("f32", 8, 64, 8), ("bf16", 5, 128, 4),
                                          ("f16", 2, 128, 8), ("f32", 1, 64, 32),
                                          ("bf16", 4, 128, 64), ("f16", 8, 64, 64),
                                          ("f32", 2, 64, 64)])
def test_shapes_and_ragged_lengths(dtype, G, D, bs):
    lens = [0, 1, 15, 16, 17, 63, 64, 65, 127, 511, 512, 513, 1100]
    wl = workloads.custom(f"ragged", lens, 2 * G, 2, D, dtype, bs, 4096 // bs * 4, seed=5,
                          steps=0)
    errs, _, _ = run_parity(wl, table_width=1100 // bs + 2, partition_size=128)
    assert max(errs) <= TOL[dtype], errs


def test_variants_and_partitions_agree():
    pa = _pa()
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    wl = workloads.custom("agree", [3000, 17, 640, 1], 16, 2, 128, "bf16", 16, 512, seed=7,
                          steps=1)
    steps = list(wl.steps)
    outs = []
    for variant, part in ((1, 64), (1, 1024), (2, 64), (2, 512), (2, 1024), (3, 64), (3, 512),
                          (3, 1024)):
        r = PagedKVRunner.for_shape(wl.shape, 200, partition_size=part, variant=variant)
        out = None
        for st in steps:
            o = r.run(st)
            out = o if o is not None else out
        outs.append(out.cpu())
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 2 * TOL["bf16"]


def test_empty_batch_and_zero_lengths():
    pa = _pa()
    kc = torch.zeros(4, 2, 16, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.randn(3, 4, 128, device="cuda").to(torch.bfloat16)
    out = torch.full((3, 4, 128), 7.0, device="cuda")
    bt = torch.zeros(3, 2, dtype=torch.int32, device="cuda")
    sl = torch.zeros(3, dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, kc, kc.clone(), bt, sl, 0.1)
    assert torch.all(out == 0)
    pa.pa_decode(out[:0], q[:0], kc, kc.clone(), bt[:0], sl[:0], 0.1)


def test_device_checks_flag_bad_tables_and_lengths():
    pa = _pa()
    pa.device_errors(clear=True)
    kc = torch.randn(4, 1, 16, 128, device="cuda").to(torch.bfloat16)
    q = torch.randn(2, 2, 128, device="cuda").to(torch.bfloat16)
    out = torch.empty(2, 2, 128, device="cuda")
    bt = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device="cuda")   # 9 >= NB
    sl = torch.tensor([20, 5], dtype=torch.int32, device="cuda")
    for variant in (1, 2):
        pa.pa_decode(out, q, kc, kc.clone(), bt, sl, 0.1, variant=variant)
        assert pa.device_errors(clear=True) == ["table"]
    sl = torch.tensor([40, 5], dtype=torch.int32, device="cuda")            # 40 > 2 blocks
    for variant in (1, 2):
        pa.pa_decode(out, q, kc, kc.clone(), bt, sl, 0.1, variant=variant)
        assert pa.device_errors(clear=True) == ["seqlen"]
        assert torch.all(out[0] == 0)


def test_profile_events_bracket_the_main_kernel():
    pa = _pa()
    wl = workloads.custom("prof", [2048] * 4, 32, 8, 128, "bf16", 16, 1024, seed=3, steps=1)
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    r = PagedKVRunner.for_shape(wl.shape, 128)
    steps = list(wl.steps)
    r.run(steps[0])
    b, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pa.set_profile_events(b, e)
    r.run(steps[1])
    pa.set_profile_events(None, None)
    torch.cuda.synchronize()
    assert b.elapsed_time(e) > 0


def test_pinned_host_fed_steps_match_oracle():
    """The host-fed step path (one packed copy of slots/tables/lengths, inputs
    from pinned memory, output read back) gives the oracle's outputs."""
    from oracle.run import OracleRun
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    wl = workloads.beam(steps=3, groups=2, beams=3, prefix=70, num_blocks=128)
    orc = OracleRun(wl.shape)
    r = PagedKVRunner.for_shape(wl.shape, 16)
    for i, st in enumerate(wl.steps):
        ref = orc.step(st)
        if st.q is None:
            r.run(st)
            continue
        out = torch.empty((st.q.shape[0], wl.shape.num_heads, wl.shape.head_dim)).pin_memory()
        res = r.run_pinned(st.ops, st.k_new.pin_memory(), st.v_new.pin_memory(),
                           st.q.pin_memory(), out)
        assert res["h2d"] > 0 and res["d2h"] == out.nbytes
        err = float(np.abs(out.double().numpy() - ref["out"]).max())
        assert err <= TOL["f16"], (i, err)


def test_prefix_cached_requests_decode_like_the_oracle():
    """Requests sharing a cached system prompt reuse its blocks (fewer rows
    written) and decode exactly as if each had its own copy."""
    wl = workloads.prefix_share(requests=8, prompt=300, suffix_hi=40, steps=3)
    errs, gpu, orc = run_parity(wl, table_width=32, compare_cache=True)
    assert max(errs) <= TOL["bf16"], errs
    st = gpu.alloc.stats()
    assert st["prefix_hit_blocks"] == 7 * (300 // 16) == orc.alloc.stats()["prefix_hit_blocks"]


def test_preempted_sequence_swaps_out_and_back_and_decodes_on():
    wl = workloads.preempt(batch=4, lo=100, hi=600, steps=6, host_blocks=64, num_blocks=256)
    errs, gpu, orc = run_parity(wl, table_width=48, compare_cache=True)
    assert len(errs) == 6 and max(errs) <= TOL["bf16"], errs
    # the victim's rows came back from host blocks into fresh device blocks
    assert gpu.alloc.stats()["swapped_seqs"] == 0 and gpu.alloc.stats()["host_free_blocks"] == 64


# ---------------------------------------------------------------- chunked prefill
# prefill_variant 1 = mma.sync kernel, 2 = tcgen05 kernel (TMEM accumulators),
# 3 = the tcgen05 kernel persistent (one CTA per SM walking its share of the tiles)
@pytest.mark.parametrize("pv", [1, 2, 3])
@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", [("bf16", 32, 8, 128, 16), ("f16", 8, 8, 64, 8),
                                               ("bf16", 16, 2, 128, 32), ("bf16", 6, 2, 64, 64),
                                               ("f16", 12, 2, 128, 16), ("bf16", 7, 7, 128, 8)])
def test_chunked_prefill_matches_oracle(dtype, Hq, Hkv, D, bs, pv):
    wl = workloads.chunked_prefill(batch=5, ctx_lo=0, ctx_hi=400, chunk_lo=1, chunk_hi=200,
                                   num_heads=Hq, num_kv_heads=Hkv, head_dim=D, dtype=dtype,
                                   block_size=bs, num_blocks=4096 // bs * 2, chunks=2)
    errs, _, _ = run_parity(wl, table_width=1000 // bs + 2, prefill_variant=pv)
    assert len(errs) == 2 and max(errs) <= TOL[dtype], errs


# prefill_variant 4: the tcgen05 kernel with P entering the PV product as one
# fp16 per weight (a bf16 cache's V stages converted to fp16 in shared memory)
@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", [("f16", 8, 8, 64, 8), ("f16", 12, 2, 128, 16),
                                               ("bf16", 32, 8, 128, 16), ("bf16", 6, 2, 64, 64),
                                               ("bf16", 7, 7, 128, 32), ("bf16", 16, 2, 128, 8),
                                               ("f16", 32, 8, 128, 16)])
def test_chunked_prefill_one_fp16_p_matches_oracle(dtype, Hq, Hkv, D, bs):
    wl = workloads.chunked_prefill(batch=5, ctx_lo=0, ctx_hi=400, chunk_lo=1, chunk_hi=200,
                                   num_heads=Hq, num_kv_heads=Hkv, head_dim=D, dtype=dtype,
                                   block_size=bs, num_blocks=4096 // bs * 2, chunks=2)
    errs, _, _ = run_parity(wl, table_width=1000 // bs + 2, prefill_variant=4)
    assert len(errs) == 2 and max(errs) <= TOL[dtype], errs


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_prefill_one_fp16_p_long_context_sampled(dtype):
    """Variant 4 on the prefill study's first shape (8 x (4096 + 1024),
    32/8 heads, D 128, bs 16): 64 sampled (row, head) pairs."""
    wl = workloads.chunked_prefill(batch=8, ctx_lo=4096, ctx_hi=4096, chunk_lo=1024,
                                   chunk_hi=1024, dtype=dtype,
                                   num_blocks=8 * (4096 + 1024) // 16 + 64)
    errs, _, _ = run_parity(wl, table_width=(4096 + 1024) // 16 + 2, sample=64,
                            prefill_variant=4)
    assert len(errs) == 1 and max(errs) <= TOL[dtype], errs


def test_prefill_one_fp16_p_edge_shapes():
    """Variant 4: empty chunks beside 1-3-token ones, and G = 5 with idle rows."""
    for Hq, Hkv, ctx, lo, hi in ((16, 4, 300, 0, 3), (10, 2, 500, 1, 300)):
        wl = workloads.chunked_prefill(seed=11, batch=6, ctx_lo=ctx // 2, ctx_hi=ctx,
                                       chunk_lo=lo, chunk_hi=hi, num_heads=Hq, num_kv_heads=Hkv,
                                       head_dim=128, dtype="bf16", block_size=16,
                                       num_blocks=6 * (ctx + 2 * hi) // 16 + 64, chunks=2)
        errs, _, _ = run_parity(wl, table_width=(ctx + 2 * hi) // 16 + 2, prefill_variant=4)
        assert len(errs) == 2 and max(errs) <= TOL["bf16"], errs


def test_prefill_one_fp16_p_reports_values_beyond_fp16():
    """A bf16 V value of 1e5 has no fp16 counterpart: variant 4 sets the
    "range" device error bit (its tile's rows are not finite); variant 2
    computes the same call within tolerance of the oracle."""
    from oracle import attn
    pa = _pa()
    pa.device_errors()
    g = torch.Generator().manual_seed(5)
    Hkv, G, D, bs, L, n = 2, 4, 128, 16, 200, 40
    nb = (L + bs - 1) // bs
    kc = torch.randn(nb, Hkv, bs, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(nb, Hkv, bs, D, generator=g).to(torch.bfloat16)
    vc[3, 1, 5, 7] = 1e5
    q = torch.randn(n, Hkv * G, D, generator=g).to(torch.bfloat16)
    tab = torch.arange(nb, dtype=torch.int32).view(1, nb)
    sl = torch.tensor([L], dtype=torch.int32)
    cu = torch.tensor([0, n], dtype=torch.int32)
    exp = attn.paged_prefill(q, kc, vc, tab.numpy(), sl.numpy(), cu.numpy(), 0.088)
    out = torch.empty(n, Hkv * G, D, dtype=torch.float32, device="cuda")
    args = (q.cuda(), kc.cuda(), vc.cuda(), tab.cuda(), sl.cuda(), cu.cuda(), 0.088)
    pa.pa_prefill(out, *args[:6], args[6], max_q_len=n, variant=4)
    assert pa.device_errors() == ["range"]
    got = out.double().cpu().numpy()
    assert not np.isfinite(got[:, G:, 7]).any()  # KV head 1's rows, that column
    assert float(np.abs(got[:, :G] - exp[:, :G]).max()) <= 3e-3  # KV head 0: unaffected
    pa.pa_prefill(out, *args[:6], args[6], max_q_len=n, variant=2)
    assert pa.device_errors() == []
    got = out.double().cpu().numpy()
    assert float(np.abs(got[:, :G] - exp[:, :G]).max()) <= 3e-3
    # variant 2 carries P to within 2^-14 of each weight: an error bound
    # proportional to the largest |v|
    assert float(np.abs(got[:, G:] - exp[:, G:]).max()) <= 2.0 ** -13 * 1e5


@pytest.mark.parametrize("pv", [1, 2, 3])
def test_chunk_covering_the_whole_sequence_and_single_tokens(pv):
    wl = workloads.chunked_prefill(batch=6, ctx_lo=0, ctx_hi=0, chunk_lo=1, chunk_hi=130,
                                   num_blocks=512, chunks=3)
    errs, _, _ = run_parity(wl, table_width=32, prefill_variant=pv)
    assert max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("pv", [1, 2, 3])
def test_prefill_long_context(pv):
    """Chunks of 512-1024 rows after 2k-6k tokens of context: many 64-key
    stages per CTA, several CTAs per sequence, ragged last CTA and stage."""
    wl = workloads.chunked_prefill(batch=2, ctx_lo=2000, ctx_hi=4000, chunk_lo=512,
                                   chunk_hi=1024, num_heads=16, num_kv_heads=4, head_dim=128,
                                   dtype="bf16", block_size=16, num_blocks=1024, chunks=1)
    errs, _, _ = run_parity(wl, table_width=5100 // 16 + 2, prefill_variant=pv)
    assert max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("pv", [1, 2, 3])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("scale", [-0.2, 0.0, 0.5])
def test_prefill_any_finite_scale(pv, dtype, scale):
    """The logit scale is any finite number: negative scales reverse the
    softmax order, 0 gives the plain mean of the attended values."""
    from oracle import attn
    from oracle.run import OracleRun
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    pa = _pa()
    wl = workloads.chunked_prefill(batch=3, ctx_lo=100, ctx_hi=300, chunk_lo=1, chunk_hi=160,
                                   num_heads=8, num_kv_heads=2, head_dim=128, dtype=dtype,
                                   block_size=16, num_blocks=256, chunks=1)
    sh = wl.shape
    orc, gpu = OracleRun(sh), PagedKVRunner.for_shape(sh, 32)
    for st in wl.steps:
        ref = orc.step(st, decode=False)
        acts = gpu.plan(st.ops)
        gpu.upload(acts)
        gpu.execute(acts, st.k_new.cuda(), st.v_new.cuda(),
                    None if st.q is None else st.q.cuda())
    a = [x for x in acts if x.kind == "prefill"][0]
    q = st.q
    out = torch.empty((q.shape[0], sh.num_heads, sh.head_dim), dtype=torch.float32,
                      device="cuda")
    pa.pa_prefill(out, q.cuda(), gpu.k_cache, gpu.v_cache, a.dev["tables"], a.dev["lens"],
                  a.dev["cu"], scale, max_q_len=a.max_q, max_seq_len=a.max_len, variant=pv)
    exp = attn.paged_prefill(q, orc.k_cache, orc.v_cache, ref["block_tables"],
                             ref["seq_lens"], a.cu, scale)
    err = float(np.abs(out.double().cpu().numpy() - exp).max())
    assert err <= TOL[dtype], err


# ---------------------------------------------------------------- graph replay
def test_graph_replayed_steps_match_the_oracle():
    """Decode steps fed from page-locked host memory and replayed from CUDA
    graphs (PagedKVRunner.launch_graph: one capture per staging slot, then
    replays with new allocator output, K/V rows and queries) give the oracle's
    output at every step; the lengths cross block and 512-token split edges."""
    from oracle.run import OracleRun
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    wl = workloads.custom("graph", [700, 33, 1, 510], 16, 4, 128, "bf16", 16, 256, seed=5,
                          steps=7)
    steps = list(wl.steps)
    orc, gpu = OracleRun(wl.shape), PagedKVRunner.for_shape(wl.shape, 48)
    orc.step(steps[0])
    gpu.run(steps[0])
    replays = 0
    for n, st in enumerate(steps[1:]):
        if n == 3:
            # a larger eager decode grows the binding's workspace; the graphs
            # captured before keep writing into the buffer they were given
            pa = _pa()
            big = torch.zeros(64, 4, 16, 128, dtype=torch.bfloat16, device="cuda")
            q = torch.zeros(64, 32, 128, dtype=torch.bfloat16, device="cuda")
            out = torch.empty(64, 32, 128, dtype=torch.float32, device="cuda")
            tables = torch.zeros(64, 2048, dtype=torch.int32, device="cuda")
            lens = torch.full((64,), 16, dtype=torch.int32, device="cuda")
            pa.pa_decode(out, q, big, big, tables, lens, 0.1, max_seq_len=32768)
            torch.cuda.synchronize()
        ref = orc.step(st)
        prep = gpu.prepare(st.ops)
        res = gpu.launch_graph(prep, st.k_new.pin_memory(), st.v_new.pin_memory(),
                               st.q.pin_memory())
        assert res is not None, "a plain append + decode step has a graph form"
        gpu.wait()
        err = float(np.abs(res["out"].double().numpy() - ref["out"]).max())
        assert err <= TOL["bf16"], err
        replays += 1
    assert replays == 7
    # a copy-on-write step has no graph form: nothing is launched
    gpu.alloc.seq_fork(0, 99)
    prep = gpu.prepare([("append", 0, 1), ("decode", [0, 99])])
    assert gpu.launch_graph(prep, torch.zeros(1, 4, 128, dtype=torch.bfloat16).pin_memory(),
                            torch.zeros(1, 4, 128, dtype=torch.bfloat16).pin_memory(),
                            torch.zeros(2, 16, 128, dtype=torch.bfloat16).pin_memory()) is None


def test_steps_read_one_step_behind_match_the_oracle():
    """The benchmark's pipelined loop: step i+1 is prepared, staged and
    launched before the host waits for step i's output, graph steps and eager
    (copy-on-write) steps mixed; every output, read one step late, is the
    oracle's for its own step."""
    from oracle.run import OracleRun
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    wl = workloads.custom("pipe", [700, 33, 1, 510], 16, 4, 128, "bf16", 16, 256, seed=6,
                          steps=8)
    steps = list(wl.steps)
    orc, gpu = OracleRun(wl.shape), PagedKVRunner.for_shape(wl.shape, 48)
    orc.step(steps[0])
    gpu.run(steps[0])
    refs = [orc.step(st)["out"] for st in steps[1:]]
    host = [(st.ops, st.k_new.pin_memory(), st.v_new.pin_memory(), st.q.pin_memory())
            for st in steps[1:]]
    outs = [torch.empty(tuple(refs[0].shape), dtype=torch.float32).pin_memory() for _ in range(2)]
    got, pending, kinds = [], [], []
    prep = gpu.prepare(host[0][0])
    gr = gpu.stage_graph(prep, *host[0][1:]) if 0 % 3 else None
    for i in range(len(host)):
        if gr is not None:
            res = gpu.replay_graph(gr, prep)
            kinds.append("graph")
        else:
            res = gpu.launch(prep, *host[i][1:], outs[i & 1])
            res["out"] = outs[i & 1]
            kinds.append("eager")
        ev = res.get("ready")  # a graph step's output copy runs on its own stream
        if ev is None:
            ev = torch.cuda.Event()
            ev.record()
        pending.append((ev, res))
        if len(pending) > 1:
            e, r = pending.pop(0)
            e.synchronize()
            got.append(r["out"].double().numpy().copy())
        if i + 1 < len(host):
            prep = gpu.prepare(host[i + 1][0])
            # every third step launches eagerly, the rest replay graphs
            gr = gpu.stage_graph(prep, *host[i + 1][1:]) if (i + 1) % 3 else None
    e, r = pending.pop(0)
    e.synchronize()
    got.append(r["out"].double().numpy().copy())
    assert "graph" in kinds and "eager" in kinds
    for i, (g, ref) in enumerate(zip(got, refs)):
        err = float(np.abs(g - ref).max())
        assert err <= TOL["bf16"], (i, kinds[i], err)


@pytest.mark.parametrize("pv", [1, 2, 3])
@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs,ctx,chunk_lo,chunk_hi", [
    ("bf16", 16, 4, 128, 16, 300, 0, 3),     # empty chunks next to 1-3-token ones (seed 11)
    ("bf16", 10, 2, 128, 16, 500, 1, 300),   # G = 5: 25 tokens x 5 heads + 3 idle rows per tile
    ("f16", 8, 2, 64, 64, 3000, 200, 700),   # 64-token blocks, D 64, 3000-token context
])
def test_prefill_edge_shapes(pv, dtype, Hq, Hkv, D, bs, ctx, chunk_lo, chunk_hi):
    wl = workloads.chunked_prefill(seed=11, batch=6, ctx_lo=ctx // 2, ctx_hi=ctx,
                                   chunk_lo=chunk_lo, chunk_hi=chunk_hi, num_heads=Hq,
                                   num_kv_heads=Hkv, head_dim=D, dtype=dtype, block_size=bs,
                                   num_blocks=6 * (ctx + 2 * chunk_hi) // bs + 64, chunks=2)
    errs, _, _ = run_parity(wl, table_width=(ctx + 2 * chunk_hi) // bs + 2, prefill_variant=pv)
    assert len(errs) == 2 and max(errs) <= TOL[dtype], errs


@pytest.mark.parametrize("pv", [2, 3])
def test_prefill_many_tiles_per_cta(pv):
    """Forty sequences with chunks of 0 to 300 tokens after 0 to 700 tokens of
    context: ~800 token tiles (many of them empty) for 148 persistent CTAs,
    so every CTA walks several tiles of different sequences and lengths, with
    empty ones skipped between them, in both of its Q buffers."""
    wl = workloads.chunked_prefill(seed=13, batch=40, ctx_lo=0, ctx_hi=700, chunk_lo=0,
                                   chunk_hi=300, num_heads=16, num_kv_heads=4, head_dim=128,
                                   dtype="bf16", block_size=16,
                                   num_blocks=40 * (700 + 600) // 16 + 64, chunks=2)
    errs, _, _ = run_parity(wl, table_width=(700 + 600) // 16 + 2, prefill_variant=pv)
    assert len(errs) == 2 and max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("pv", [1, 2, 3])
def test_prefill_full_study_size_sampled(pv):
    """The prefill study's first workload at full size (8 sequences, 4096
    tokens of context + a 1024-token chunk, 32/8 heads, D 128, bf16, bs 16),
    in the launch configuration the study times; 64 sampled (row, head) pairs,
    the first and the last row among them, against the fp64 oracle."""
    wl = workloads.chunked_prefill(batch=8, ctx_lo=4096, ctx_hi=4096, chunk_lo=1024,
                                   chunk_hi=1024, num_blocks=8 * (4096 + 1024) // 16 + 64)
    errs, _, _ = run_parity(wl, table_width=(4096 + 1024) // 16 + 2, sample=64,
                            prefill_variant=pv)
    assert len(errs) == 1 and max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("pv", [1, 2, 3])
def test_prefill_bad_table_entry_is_reported(pv):
    """A table entry outside [0, num_blocks) is read as zeros and sets the
    "table" device error bit; the other sequences still match the oracle."""
    from oracle import attn
    from oracle.run import OracleRun
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    pa = _pa()
    wl = workloads.chunked_prefill(batch=3, ctx_lo=100, ctx_hi=200, chunk_lo=20, chunk_hi=80,
                                   num_heads=8, num_kv_heads=2, head_dim=128, dtype="bf16",
                                   block_size=16, num_blocks=128, chunks=1)
    sh = wl.shape
    orc, gpu = OracleRun(sh), PagedKVRunner.for_shape(sh, 24)
    for st in wl.steps:
        ref = orc.step(st)
        acts = gpu.plan(st.ops)
        gpu.upload(acts)
        gpu.execute(acts, st.k_new.cuda(), st.v_new.cuda(),
                    None if st.q is None else st.q.cuda())
    a = [x for x in acts if x.kind == "prefill"][0]
    tables = a.dev["tables"].clone()
    tables[0, 1] = sh.num_blocks + 5  # sequence 0's second block
    out = torch.empty((st.q.shape[0], sh.num_heads, sh.head_dim), dtype=torch.float32,
                      device="cuda")
    pa.device_errors(clear=True)
    pa.pa_prefill(out, st.q.cuda(), gpu.k_cache, gpu.v_cache, tables, a.dev["lens"],
                  a.dev["cu"], sh.scale, max_q_len=a.max_q, max_seq_len=a.max_len, variant=pv)
    torch.cuda.synchronize()
    assert pa.device_errors(clear=True) == ["table"]
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    rows = slice(int(a.cu[1]), int(a.cu[-1]))  # sequences 1 and 2 are untouched
    assert float(np.abs(got[rows] - ref["out"][rows]).max()) <= TOL["bf16"]
