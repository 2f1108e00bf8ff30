"""The C ABI library loads without a GPU and exports what the header declares;
argument checks that need no device return their status codes."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from conftest import ROOT


def _declared():
    src = open(os.path.join(ROOT, "include", "pagedattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_copy_blocks", "pa_alloc_create",
              "pa_seq_append", "pa_seq_fork", "pa_seq_free", "pa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from paged_kv_cache_347_b200 import pagedattn as pa
    lib = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert pa.version() >= 10000


def test_binding_names_every_device_error_bit():
    """The binding's names for the device error word cover exactly the bits
    the header defines."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    src = open(os.path.join(ROOT, "include", "pagedattn.h")).read()
    bits = {int(v, 16): n.lower()
            for n, v in re.findall(r"#define PA_DEVERR_([A-Z]+)\s+(0x[0-9a-fA-F]+)u", src)}
    assert bits == pa.DEVERR


def test_checks_before_any_device_work():
    from paged_kv_cache_347_b200 import pagedattn as pa
    L = pa._lib
    # unsupported head_dim / block_size / dtype / GQA group
    args = dict(out=None, q=None, kc=None, vc=None, bt=None, sl=None)
    rc = L.pa_decode(None, None, None, None, None, None, 1, 8, 8, 96, 16, 4, 64, 64, 1.0, 1,
                     None, 0, None)
    assert rc == -2
    rc = L.pa_decode(None, None, None, None, None, None, 1, 8, 8, 128, 12, 4, 64, 48, 1.0, 1,
                     None, 0, None)
    assert rc == -2 and b"block_size" in L.pa_last_error()
    rc = L.pa_decode(None, None, None, None, None, None, 1, 18, 2, 128, 16, 4, 64, 64, 1.0, 1,
                     None, 0, None)
    assert rc == -2 and b"GQA" in L.pa_last_error()
    rc = L.pa_decode(None, None, None, None, None, None, 1, 8, 8, 128, 16, 4, 64, 64, 1.0, 7,
                     None, 0, None)
    assert rc == -2
    # max_seq_len beyond the table, bad partition, NULL pointers
    rc = L.pa_decode(None, None, None, None, None, None, 1, 8, 8, 128, 16, 4, 64, 65, 1.0, 1,
                     None, 0, None)
    assert rc == -1
    rc = L.pa_decode_ex(None, None, None, None, None, None, 1, 8, 8, 128, 16, 4, 64, 64, 1.0, 1,
                        None, 0, 100, 0, None)
    assert rc == -1 and b"partition" in L.pa_last_error()
    rc = L.pa_decode(None, None, None, None, None, None, 1, 8, 8, 128, 16, 4, 64, 64, 1.0, 1,
                     None, 0, None)
    assert rc == -1 and b"NULL" in L.pa_last_error()
    # the tensor-core kernel does not take fp32
    rc = L.pa_decode_ex(None, None, None, None, None, None, 1, 8, 8, 128, 16, 4, 64, 64, 1.0, 0,
                        None, 0, 0, 2, None)
    assert rc == -2
    # nothing to do is success without a device
    assert L.pa_decode(None, None, None, None, None, None, 0, 8, 8, 128, 16, 4, 64, 64, 1.0, 1,
                       None, 0, None) == 0
    assert L.pa_reshape_and_cache(None, None, None, None, None, 0, 8, 128, 16, 64, 1, None) == 0
    assert L.pa_copy_blocks(None, None, None, 0, 4096, 64, None) == 0
    assert L.pa_copy_blocks(1, 1, 8, 1, 15, 64, None) == -1
    assert L.pa_reshape_and_cache(None, None, None, None, None, 3, 8, 128, 16, 64, 1, None) == -1


def test_workspace_size():
    from paged_kv_cache_347_b200 import pagedattn as pa
    assert pa.decode_workspace_size(8, 64, 128, 512) == 0
    n = pa.decode_workspace_size(8, 64, 128, 32768)
    units = 8 * 64 * 64
    # partials, then one 8-byte merge ticket per (sequence, head)
    assert n == units * 128 * 4 + units * 2 * 4 + 8 * 64 * 8
    assert pa.decode_workspace_size(8, 64, 128, 32768, 1024) < n
    # a length bound near INT_MAX: the split count is formed in 64 bits
    big = 2 ** 31 - 1
    splits = -(-big // 512)
    assert pa.decode_workspace_size(1, 1, 128, big) == (
        -(-splits * 128 * 4 // 256) * 256 + -(-splits * 2 * 4 // 256) * 256 + 256)


def test_python_binding_rejects_cpu_tensors():
    from paged_kv_cache_347_b200 import pagedattn as pa
    kc = torch.zeros(4, 1, 16, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        pa.pa_reshape_and_cache(torch.zeros(1, 1, 128, dtype=torch.bfloat16),
                                torch.zeros(1, 1, 128, dtype=torch.bfloat16), kc, kc.clone(),
                                torch.zeros(1, dtype=torch.int64))


def test_selftest_wait_rejects_bad_arguments_before_any_cuda_call():
    from paged_kv_cache_347_b200 import pagedattn as pa
    invalid = -1  # PA_ERR_INVALID_ARG
    assert pa._lib.pa_selftest_wait(0, 0, None, None) == invalid
    assert pa._lib.pa_selftest_wait(10**11, 0, None, None) == invalid
    assert pa._lib.pa_selftest_wait(10**6, 0, None, None) == invalid  # NULL elapsed


def _ctas(lens, part, hkv):
    return hkv * sum(1 if L == 0 else -(-int(L) // part) for L in lens)


@pytest.mark.parametrize("lens,slots", [
    ([3000] * 32, 888),                       # 6 splits x 32 x 8 = 1536 CTAs at 512: 1.7 waves
    ([3000] * 50, 888),                       # 2400 CTAs: 2.7 waves, keeps 512
    ([4000] * 20, 700),                       # 1280 at 512, 640 at 1024
    ([2048] * 32, 888),                       # 1024 CTAs at 512: one CTA past a full wave
    ([32768] * 2, 888),
    ([32768] * 8, 888),                       # 4096 CTAs: many waves, keeps 512
    ([1024] * 32, 888),                       # 512 CTAs: one wave, keeps 512
    ([0, 1, 511, 512, 513, 4096, 4097] * 20, 700),
    (list(range(0, 9000, 37)), 1000),
    ([600, 1300] * 16, 888),                  # longest > 2 x shortest
    ([600, 1100] * 200, 888),                 # within 2x, many waves: 512
    ([100, 400] * 64, 888),                   # varied but nothing past 512: 512
])
def test_partition_choice_follows_its_rule(lens, slots):
    """pa_decode_partition_for against its stated rule, evaluated here by
    brute force: 1024 when 512-token CTAs fill more than one wave and at most
    two and 1024-token ones fit one wave, or when the longest sequence is past
    512 tokens and more than twice the shortest; else 512."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    hkv = 8
    got = pa.decode_partition_for(lens, hkv, 128, 16, torch.bfloat16, slots=slots)
    n0 = _ctas(lens, 512, hkv)
    waves = slots < n0 <= 2 * slots and _ctas(lens, 1024, hkv) <= slots
    varied = max(lens) > 512 and max(lens) > 2 * min(lens)
    want = 1024 if waves or varied else 512
    assert got == want


def test_partition_choice_edge_cases():
    from paged_kv_cache_347_b200 import pagedattn as pa
    # the CUDA-core kernel (fp32 caches) keeps 512
    assert pa.decode_partition_for([2048] * 32, 8, 128, 16, torch.float32, slots=888) == 512
    # 4-row blocks of 16-bit caches take the tensor-core kernel and its rule:
    # 1024 CTAs of 512 tokens fill 1.15 waves of 888, those of 1024 fit one
    assert pa.decode_partition_for([2048] * 32, 8, 128, 4, torch.bfloat16, slots=888) == 1024
    assert pa.decode_partition_for([], 8, 128, 16, torch.bfloat16, slots=888) == 512
    with pytest.raises(pa.PagedAttnError):
        pa.decode_partition_for([5, -1], 8, 128, 16, torch.bfloat16, slots=888)
    with pytest.raises(pa.PagedAttnError):
        pa.decode_partition_for([5], 8, 100, 16, torch.bfloat16, slots=888)
    with pytest.raises(pa.PagedAttnError):
        pa.decode_partition_for([5], 8, 128, 16, torch.bfloat16, slots=-1)
    assert pa._lib.pa_decode_partition_for(None, 2, 8, 128, 16, 1, 888) == -1


def test_step_launch_rejects_bad_arguments_before_any_cuda_call():
    from paged_kv_cache_347_b200 import pagedattn as pa
    L = pa._lib
    # no event or graph
    assert L.pa_step_launch(None, None, None, None, 0, None, None, None, None, None, None,
                            None) == -1
    # a negative copy count, or copies without a list
    assert L.pa_step_launch(None, None, None, None, -1, None, 1, 1, None, 1, None, None) == -1
    assert L.pa_step_launch(None, None, None, None, 2, None, 1, 1, None, 1, None, None) == -1
    # an output graph without its event
    assert L.pa_step_launch(None, None, None, None, 0, None, 1, 1, None, 1, 1, None) == -1


def _choice_by_rule(lens, hkv, slots):
    """pa_decode_choose's rule for two-head CTAs, evaluated here by brute force."""
    def ctas(p):
        return (hkv // 2) * sum(1 if L <= p else -(-L // p) for L in lens)
    for p in (256, 384, 512, 640, 768, 1024):
        if ctas(p) <= 0.85 * slots:
            return p
    return 1024 if ctas(1024) <= slots else 512


@pytest.mark.parametrize("lens", [
    [32768] * 8,                                   # many waves at any split: 512
    [32768] * 6,                                   # 1024-token splits: 0.86 of a wave
    [2070] * 16,                                   # beam-shaped: 256
    list(np.random.default_rng(1).integers(512, 4097, 32)),    # Llama-8B-shaped
    list(np.random.default_rng(2).integers(512, 4097, 64)),
    [150] * 256,                                   # 1024 one-split CTAs: 512
    [100, 30],                                     # tiny: 256
    [0, 1, 511, 512, 513, 4096, 4097] * 20,
])
def test_decode_choice_follows_its_rule(lens):
    """pa_decode_choose: for 16-bit caches with block size 8 or 16 and an even
    KV head count, two-head CTAs (variant 3) with the split the wave rule
    gives; otherwise variant 2 (fp32: 1) with pa_decode_partition_for's split."""
    from paged_kv_cache_347_b200 import pagedattn as pa
    lens = [int(x) for x in lens]
    bf = torch.bfloat16
    for bs in (8, 16):
        assert pa.decode_choose(lens, 8, 128, bs, bf, slots=888) == (
            _choice_by_rule(lens, 8, 888), 3, 2)
    for bs in (4, 32, 64):
        assert pa.decode_choose(lens, 8, 128, bs, bf, slots=888) == (
            pa.decode_partition_for(lens, 8, 128, bs, bf, slots=888), 2, 0)
    assert pa.decode_choose(lens, 7, 128, 16, bf, slots=888)[1:] == (2, 0)
    assert pa.decode_choose(lens, 8, 128, 16, torch.float32, slots=888)[1:] == (1, 0)


def test_decode_choice_on_the_bench_shapes():
    from paged_kv_cache_347_b200 import pagedattn as pa
    bf = torch.bfloat16
    assert pa.decode_choose([32768] * 8, 8, 128, 16, bf, slots=888) == (512, 3, 2)
    assert pa.decode_choose([2070] * 16, 8, 128, 16, bf, slots=888) == (256, 3, 2)
    llama = [int(x) for x in np.random.default_rng(1).integers(512, 4097, 32)]
    assert pa.decode_choose(llama, 8, 128, 16, bf, slots=888) == (512, 3, 2)
