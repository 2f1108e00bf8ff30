"""pa_decode_static, the decode entry point for callers that cannot allocate
device memory (its split partials live in the library's fixed device array),
must give the same outputs as pa_decode with a caller workspace.

Called through the C ABI (ctypes) twice in a row with different inputs, so a
second call cannot lean on what the first left in the shared array.  Kept in
a file of its own that pytest collects last."""
import ctypes

import numpy as np
import pytest
import torch

from parity import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_347_b200 import pagedattn
    pagedattn.device_errors(clear=True)
    yield pagedattn
    assert pagedattn.device_errors(clear=True) == []


def _case(seed, B, Hq, Hkv, D, bs, lens, dtype):
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = max(-(-L // bs) for L in lens)
    NB = B * W + 7
    kc = torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(dtype)
    vc = torch.randn(NB, Hkv, bs, D, generator=g, device="cuda").to(dtype)
    perm = torch.randperm(NB, generator=g, device="cuda")[: B * W]
    tables = perm.reshape(B, W).to(torch.int32).contiguous()
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q = torch.randn(B, Hq, D, generator=g, device="cuda").to(dtype)
    return q, kc, vc, tables, sl, W * bs


def _static(pa, out, q, kc, vc, tables, sl, max_len, scale):
    NB, Hkv, bs, D = kc.shape
    B, Hq, _ = q.shape
    return pa._lib.pa_decode_static(
        out.data_ptr(), q.data_ptr(), kc.data_ptr(), vc.data_ptr(), tables.data_ptr(),
        sl.data_ptr(), B, Hq, Hkv, D, bs, tables.shape[1], NB, max_len, ctypes.c_float(scale),
        pa.DTYPE_CODE[kc.dtype], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_workspace_decode_twice(pa, dtype):
    tol = TOL["f32" if dtype == torch.float32 else "bf16"]
    cases = [
        # multi-split sequences, then a different batch with fewer splits
        _case(1, 4, 32, 8, 128, 16, [4100, 1, 777, 2048], dtype),
        _case(2, 3, 16, 2, 64, 8, [1500, 513, 64], dtype),
    ]
    for q, kc, vc, tables, sl, max_len in cases:
        scale = 1.0 / q.shape[-1] ** 0.5
        ref = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        pa.pa_decode(ref, q, kc, vc, tables, sl, scale, max_seq_len=max_len)
        got = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        rc = _static(pa, got, q, kc, vc, tables, sl, max_len, scale)
        assert rc == 0, pa._lib.pa_last_error()
        torch.cuda.synchronize()
        err = (got - ref).abs().max().item()
        assert np.isfinite(err) and err <= tol, err


def test_static_call_allocates_no_device_memory(pa):
    """After a first call (which looks up the array's address), further calls
    leave the device's free memory and the caching allocator's counters
    exactly as they were: the partials go to the library's own array."""
    q, kc, vc, tables, sl, max_len = _case(4, 3, 32, 8, 128, 16, [3000, 700, 2049],
                                           torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    scale = 128 ** -0.5
    assert _static(pa, out, q, kc, vc, tables, sl, max_len, scale) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    stats0 = torch.cuda.memory_stats()
    for _ in range(3):
        assert _static(pa, out, q, kc, vc, tables, sl, max_len, scale) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    stats1 = torch.cuda.memory_stats()
    assert free1 == free0
    for key in ("allocation.all.allocated", "segment.all.allocated",
                "allocated_bytes.all.allocated"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key
    ref = torch.empty_like(out)
    pa.pa_decode(ref, q, kc, vc, tables, sl, scale, max_seq_len=max_len)
    torch.cuda.synchronize()
    assert (out - ref).abs().max().item() <= TOL["bf16"]


def test_static_scratch_rejects_oversize_requests(pa):
    q, kc, vc, tables, sl, _ = _case(3, 2, 32, 8, 128, 16, [64, 64], torch.bfloat16)
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    # 2 sequences x 32 heads x 2048 splits of 512 tokens need 68 MB > 32 MiB
    big_table = torch.zeros(2, (1 << 20) // 16, dtype=torch.int32, device="cuda")
    rc = _static(pa, out, q, kc, vc, big_table, sl, 1 << 20, 0.1)
    assert rc == -1
    assert b"static array" in pa._lib.pa_last_error()
    # a bound near INT_MAX: the split count is formed in 64 bits and the
    # request is refused before anything is launched
    rc = _static(pa, out, q, kc, vc, big_table, sl, 2 ** 31 - 1, 0.1)
    assert rc in (-1, -2), rc
    torch.cuda.synchronize()
    assert torch.all(out == 0)
