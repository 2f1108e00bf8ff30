"""pa_runtime against the fp64 oracle (needs a B200): whole workloads fed
step by step from page-locked host memory through pa_rt_step -- the
allocator's events, copy-on-write copies, appends fused into the decode or
not, admissions after the decode, graph replays -- with every output read one
step behind the launches and compared with the oracle's, and the caches and
the allocator's free list bit for bit at the end."""
import numpy as np
import pytest
import torch

from oracle.run import OracleRun
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


def _run(pa, wl, width, max_batch, max_new):
    from paged_kv_cache_347_b200.runner import PagedKVRunner
    sh = wl.shape
    dims = (sh.num_blocks, sh.num_kv_heads, sh.block_size, sh.head_dim)
    kc = torch.zeros(dims, dtype=TORCH_DT[sh.dtype], device="cuda")
    vc = torch.zeros_like(kc)
    rt = pa.Runtime(kc, vc, sh.num_heads, width, max_batch, max_new, sh.scale, sh.free_order)
    orc = OracleRun(sh)
    outs = [torch.empty((max_batch, sh.num_heads, sh.head_dim)).pin_memory() for _ in range(2)]
    pending, errs, i = [], [], 0
    for st in wl.steps:
        ref = orc.step(st)
        enc = PagedKVRunner.encode_ops(st.ops)
        assert enc is not None
        b = int(enc.decode_ids.size)
        pin = lambda t: None if t is None else t.pin_memory()
        ins = (pin(st.k_new), pin(st.v_new), pin(st.q))
        out = outs[i & 1]
        ev = rt.step(enc.events, enc.decode_ids, *ins, out if b else None)
        pending.append((ev, ref["out"], out, b, ins))
        i += 1
        while len(pending) > 1:
            e, exp, o, n, _ = pending.pop(0)
            rt.wait_event(e)
            if exp is not None:
                errs.append(float(np.abs(o[:n].double().numpy() - exp).max()))
    for e, exp, o, n, _ in pending:
        rt.wait_event(e)
        if exp is not None:
            errs.append(float(np.abs(o[:n].double().numpy() - exp).max()))
    rt.wait()
    bits = torch.int32 if sh.dtype == "f32" else torch.int16
    assert torch.equal(kc.cpu().view(bits), orc.k_cache.view(bits))
    assert torch.equal(vc.cpu().view(bits), orc.v_cache.view(bits))
    assert rt.alloc.free_list() == orc.alloc.free_list()
    return errs, rt.stats()


def test_beam_with_copy_on_write(pa):
    errs, st = _run(pa, workloads.beam(steps=18, num_blocks=1024), 152, 16, 4 * 2050)
    assert len(errs) == 18 and max(errs) <= TOL["f16"], errs
    assert st["replays"] > 0 and st["captures"] >= 1


def test_continuous_mix_admissions_after_the_decode(pa):
    wl = workloads.mix(block_size=16, steps=6, batch=48, hi=1500, pool_slots=1 << 17)
    errs, st = _run(pa, wl, 1600 // 16 + 8, 48, 48 * 1500)
    assert len(errs) == 6 and max(errs) <= TOL["bf16"], errs


def test_llama_shaped_reduced_with_graph_replays(pa):
    wl = workloads.llama(batch=8, lo=300, hi=2200, steps=8, num_blocks=2048)
    errs, st = _run(pa, wl, 2300 // 16 + 2, 8, 8 * 2200)
    assert len(errs) == 8 and max(errs) <= TOL["bf16"], errs
    assert st["replays"] >= 4


def test_tiny_fp32(pa):
    errs, st = _run(pa, workloads.tiny(), 4, 3, 64)
    assert len(errs) == 2 and max(errs) <= TOL["f32"], errs


def test_limits_are_refused_before_anything_is_applied(pa):
    sh = workloads.tiny().shape
    kc = torch.zeros((sh.num_blocks, 1, 4, 64), device="cuda")
    rt = pa.Runtime(kc, kc.clone(), 2, 4, 2, 8, sh.scale)
    before = rt.alloc.free_list()
    ev = np.array([[pa.EV_ADD, 1, 0], [pa.EV_APPEND, 1, 9]], np.int64)   # 9 > max_new_tokens 8
    with pytest.raises(pa.PagedAttnError):
        rt.step(ev, np.empty(0, np.int64), torch.zeros(9, 1, 64).pin_memory(),
                torch.zeros(9, 1, 64).pin_memory(), None, None)
    ev = np.array([[pa.EV_DECODE, 0, 0]], np.int64)
    with pytest.raises(pa.PagedAttnError):                               # 3 rows > max_batch 2
        rt.step(ev, np.array([0, 1, 2], np.int64), None, None,
                torch.zeros(3, 2, 64).pin_memory(), torch.zeros(3, 2, 64).pin_memory())
    assert rt.alloc.free_list() == before


def test_a_step_failing_in_its_plan_leaves_the_runtime_usable(pa):
    """A step whose appends need more blocks than are free fails in the
    allocator after its new rows were already on their way in: the call
    returns PA_ERR_OUT_OF_BLOCKS once those copies are done, the allocator is
    as before, and the next step decodes over exactly the rows appended by
    the steps that succeeded (checked against softmax(q K^T * scale) V in
    float64)."""
    NB, bs, D, Hq = 16, 4, 64, 2
    kc = torch.zeros((NB, 1, bs, D), device="cuda")
    vc = torch.zeros_like(kc)
    scale = 0.125
    rt = pa.Runtime(kc, vc, Hq, 4, 2, 128, scale)
    g = torch.Generator().manual_seed(3)
    rows = lambda n: torch.randn(n, 1, D, generator=g).pin_memory()
    k1, v1 = rows(8), rows(8)
    ev = np.array([[pa.EV_ADD, 1, 0], [pa.EV_APPEND, 1, 8]], np.int64)
    rt.wait_event(rt.step(ev, np.empty(0, np.int64), k1, v1, None, None))
    before = rt.alloc.free_list()
    ev = np.array([[pa.EV_APPEND, 1, 100]], np.int64)                    # 25 blocks, 14 free
    with pytest.raises(pa.PagedAttnError) as err:
        rt.step(ev, np.empty(0, np.int64), rows(100), rows(100), None, None)
    assert err.value.code == -3                                          # PA_ERR_OUT_OF_BLOCKS
    assert rt.alloc.free_list() == before
    k2, v2, q = rows(1), rows(1), torch.randn(1, Hq, D, generator=g).pin_memory()
    out = torch.empty(1, Hq, D).pin_memory()
    ev = np.array([[pa.EV_APPEND, 1, 1], [pa.EV_DECODE, 0, 0]], np.int64)
    rt.wait_event(rt.step(ev, np.array([1], np.int64), k2, v2, q, out))
    rt.wait()
    K = torch.cat([k1, k2])[:, 0].double()
    V = torch.cat([v1, v2])[:, 0].double()
    w = torch.softmax(q[0].double() @ K.T * scale, dim=-1)
    assert float((out[0].double() - w @ V).abs().max()) <= TOL["f32"]
