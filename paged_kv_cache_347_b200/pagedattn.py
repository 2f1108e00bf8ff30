"""Python binding of libpagedattn.so (include/pagedattn.h).

Argument marshalling only: torch tensors become device pointers and sizes,
the current CUDA stream is passed through, and a non-zero status becomes a
``PagedAttnError`` carrying ``pa_last_error()``.  Every step of the path runs
in the library's CUDA kernels or its C++ allocator; there is no fallback.
If the shared library is missing this module fails to import.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_347_b200.build` "
        "(nvcc, sm_100a); there is no non-CUDA implementation")

_lib = ctypes.CDLL(LIB_PATH)

PA_F32, PA_BF16, PA_F16 = 0, 1, 2
DTYPE_CODE = {torch.float32: PA_F32, torch.bfloat16: PA_BF16, torch.float16: PA_F16}
STATUS = {0: "PA_OK", -1: "PA_ERR_INVALID_ARG", -2: "PA_ERR_UNSUPPORTED",
          -3: "PA_ERR_OUT_OF_BLOCKS", -4: "PA_ERR_UNKNOWN_SEQ", -5: "PA_ERR_CUDA",
          -6: "PA_ERR_DEVICE_BOUNDS", -7: "PA_ERR_SEQ_TOO_LONG"}
DEVERR = {0x1: "table", 0x2: "seqlen", 0x4: "slot", 0x8: "pair", 0x10: "timeout",
          0x20: "range"}

_c = ctypes
_vp, _i, _i64, _sz, _f = _c.c_void_p, _c.c_int, _c.c_int64, _c.c_size_t, _c.c_float


def _sig(name, res, *args):
    fn = getattr(_lib, name)
    fn.restype = res
    fn.argtypes = list(args)
    return fn


class pa_alloc_stats_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "num_blocks", "free_blocks", "used_blocks", "shared_blocks", "num_seqs",
        "table_entries", "logical_tokens", "reserved_slots", "cached_blocks",
        "prefix_hit_blocks", "prefix_query_blocks", "evicted_blocks", "host_blocks",
        "host_free_blocks", "swapped_seqs")]


_sig("pa_last_error", _c.c_char_p)
_sig("pa_version", _i)
_sig("pa_device_errors", _i, _vp, _i)
_sig("pa_reshape_and_cache", _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp)
_sig("pa_decode_workspace_size", _sz, _i, _i, _i, _i, _i)
_sig("pa_decode", _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
     _vp, _sz, _vp)
_sig("pa_decode_ex", _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
     _vp, _sz, _i, _i, _vp)
_sig("pa_decode_partition_for", _i, _vp, _i, _i, _i, _i, _i, _i)


class pa_decode_opts(ctypes.Structure):
    _fields_ = [("partition_size", ctypes.c_int), ("variant", ctypes.c_int),
                ("merge", ctypes.c_int), ("heads_per_cta", ctypes.c_int),
                ("seq_order", ctypes.c_void_p), ("reserved", ctypes.c_int * 4)]


_sig("pa_decode_opt", _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
     _vp, _sz, _c.POINTER(pa_decode_opts), _vp)
_sig("pa_decode_choose", _i, _vp, _i, _i, _i, _i, _i, _i, _c.POINTER(pa_decode_opts))


def decode_choose(seq_lens, num_kv_heads: int, head_dim: int, block_size: int, dtype,
                  slots: int = 0) -> Tuple[int, int, int]:
    """pa_decode_choose: (partition_size, variant, heads_per_cta) for a batch
    of these host lengths."""
    lens = np.ascontiguousarray(np.asarray(seq_lens), dtype=np.int32).reshape(-1)
    code = DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    o = pa_decode_opts()
    _check(_lib.pa_decode_choose(lens.ctypes.data if lens.size else None, lens.size,
                                 num_kv_heads, head_dim, block_size, code, slots,
                                 ctypes.byref(o)), "pa_decode_choose")
    return o.partition_size, o.variant, o.heads_per_cta
_sig("pa_append_decode", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
     _i, _i, _i, _f, _i, _vp, _sz, _c.POINTER(pa_decode_opts), _vp)
_sig("pa_copy_blocks", _i, _vp, _vp, _vp, _i, _sz, _i, _vp)
_sig("pa_decode_static", _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
     _i, _vp)
_sig("pa_set_profile_events", _i, _vp, _vp)
_sig("pa_alloc_create", _i, _c.POINTER(_vp), _i, _i, _i, _vp)
_sig("pa_alloc_destroy", None, _vp)
_sig("pa_seq_add", _i, _vp, _i64)
_sig("pa_seq_append", _i, _vp, _i64, _i, _vp, _vp, _vp)
_sig("pa_batch_append", _i, _vp, _vp, _i, _vp, _vp, _vp, _vp)
_sig("pa_seq_fork", _i, _vp, _i64, _i64)
_sig("pa_seq_free", _i, _vp, _i64)
_sig("pa_seq_block_table", _i, _vp, _i64, _vp, _i, _vp, _vp)
_sig("pa_block_tables", _i, _vp, _vp, _i, _vp, _i, _vp)
_sig("pa_alloc_stats", _i, _vp, _c.POINTER(pa_alloc_stats_t))


class pa_step_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_slots", "n_slots_pre", "n_pairs", "n_pairs_pre", "num_seqs", "width",
        "max_seq_len", "events_applied")] + [(n, ctypes.c_int64) for n in (
            "off_slots", "off_pairs", "off_tables", "off_lens", "off_order", "bytes")]


_sig("pa_decode_order", _i, _vp, _i, _vp)


class pa_host_copy(ctypes.Structure):
    _fields_ = [("dst", ctypes.c_void_p), ("src", ctypes.c_void_p), ("bytes", ctypes.c_size_t)]


_sig("pa_step_launch", _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp)


def step_launch(stream_in: int, stream_run: int, stream_out: int, copies, n_copies: int,
                wait_before_in: int, event_in: int, graph_run: int, wait_before_run: int,
                event_run: int, graph_out: int, event_out: int) -> None:
    """pa_step_launch on raw handles (streams, events, graph execs as ints)."""
    _check(_lib.pa_step_launch(stream_in, stream_run, stream_out, copies, n_copies,
                               wait_before_in or None, event_in, graph_run,
                               wait_before_run or None, event_run, graph_out or None,
                               event_out or None), "pa_step_launch")


def decode_order(seq_lens) -> np.ndarray:
    """pa_decode_order: batch rows longest first (ties in batch order)."""
    lens = np.ascontiguousarray(np.asarray(seq_lens), dtype=np.int32).reshape(-1)
    out = np.empty(max(lens.size, 1), np.int32)
    _check(_lib.pa_decode_order(lens.ctypes.data if lens.size else None, lens.size,
                                out.ctypes.data), "pa_decode_order")
    return out[:lens.size]


_sig("pa_step_plan", _i, _vp, _vp, _i, _vp, _i, _i, _vp, _sz, _vp, _c.POINTER(pa_step_layout))


class pa_runtime_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "num_blocks", "block_size", "num_heads", "num_kv_heads", "head_dim", "dtype",
        "table_width", "max_batch", "max_new_tokens", "max_blocks_per_seq")] + [
        ("scale", ctypes.c_float)]


_sig("pa_rt_create", _i, _c.POINTER(_vp), _c.POINTER(pa_runtime_config), _vp, _vp, _vp)
_sig("pa_rt_destroy", None, _vp)
_sig("pa_rt_allocator", _vp, _vp)
_sig("pa_rt_step", _i, _vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _c.POINTER(_vp))
_sig("pa_rt_wait", _i, _vp)
_sig("pa_event_wait", _i, _vp)
_sig("pa_rt_stats", _i, _vp, _vp, _vp, _vp)
EV_ADD, EV_FREE, EV_FORK, EV_APPEND, EV_DECODE = 1, 2, 3, 4, 5
_sig("pa_alloc_free_list", _i, _vp, _vp, _i, _vp)
_sig("pa_alloc_refcount", _i, _vp, _i)
_sig("pa_seq_add_cached", _i, _vp, _i64, _vp, _i, _vp)
_sig("pa_seq_append_tokens", _i, _vp, _i64, _vp, _i, _vp, _vp, _vp)
_sig("pa_alloc_set_host_pool", _i, _vp, _i)
_sig("pa_seq_swap_out", _i, _vp, _i64, _vp, _i, _vp)
_sig("pa_seq_swap_in", _i, _vp, _i64, _vp, _i, _vp)
_sig("pa_swap_blocks", _i, _vp, _vp, _vp, _vp, _vp, _i, _sz, _i, _i, _vp)
_sig("pa_prefill", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i,
     _f, _i, _vp)
_sig("pa_selftest_wait", _i, _c.c_uint64, _c.c_uint64, _vp, _vp)
_sig("pa_prefill_ex", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
     _i, _f, _i, _i, _vp)


class PagedAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = _lib.pa_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS.get(code, code)}: {msg}")
        self.code = code


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise PagedAttnError(rc, where)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def version() -> int:
    return _lib.pa_version()


def device_errors(clear: bool = True) -> List[str]:
    """Names of the device error bits set since the last clear (synchronises)."""
    flags = ctypes.c_uint32(0)
    rc = _lib.pa_device_errors(ctypes.addressof(flags), 1 if clear else 0)
    if rc not in (0, -6):
        _check(rc, "pa_device_errors")
    return [n for b, n in DEVERR.items() if flags.value & b]


def set_profile_events(begin: Optional[torch.cuda.Event], end: Optional[torch.cuda.Event]) -> None:
    """Record `begin`/`end` around the main decode kernel of later pa_decode calls.

    torch creates its events lazily and only lets elapsed_time() read events it
    recorded itself, so both are recorded once here (on the current stream,
    before any later call re-records them through the library)."""
    if begin is None or end is None:
        _check(_lib.pa_set_profile_events(None, None), "pa_set_profile_events")
    else:
        begin.record()
        end.record()
        _check(_lib.pa_set_profile_events(begin.cuda_event, end.cuda_event),
               "pa_set_profile_events")


# ----------------------------------------------------------------- kernels
def pa_reshape_and_cache(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor,
                         v_cache: torch.Tensor, slot_mapping: torch.Tensor) -> None:
    """k, v [N, Hkv, D]; caches [NB, Hkv, bs, D]; slot_mapping int64 [N]."""
    NB, Hkv, bs, D = k_cache.shape
    dt = DTYPE_CODE[k_cache.dtype]
    n = slot_mapping.numel()
    if tuple(k.shape) != (n, Hkv, D) or tuple(v.shape) != (n, Hkv, D):
        raise ValueError(f"k/v must be [{n}, {Hkv}, {D}]")
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache shapes differ")
    _check(_lib.pa_reshape_and_cache(
        _dev(k, "k", k_cache.dtype), _dev(v, "v", k_cache.dtype), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache", k_cache.dtype), _dev(slot_mapping, "slot_mapping", torch.int64),
        n, Hkv, D, bs, NB, dt, _stream(k_cache)), "pa_reshape_and_cache")


_ws_cache: Dict[Tuple[int, int], torch.Tensor] = {}


def decode_workspace_size(num_seqs: int, num_heads: int, head_dim: int, max_seq_len: int,
                          partition_size: int = 0) -> int:
    return _lib.pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_seq_len,
                                         partition_size)


def decode_partition_for(seq_lens, num_kv_heads: int, head_dim: int, block_size: int,
                         dtype, slots: int = 0) -> int:
    """pa_decode_partition_for: a partition_size for pa_decode from the host
    copy of the sequence lengths (512 unless that leaves a part-empty second
    wave of CTAs).  dtype: a torch dtype or a PA_* code; slots 0 asks the
    device how many decode CTAs it holds at once."""
    lens = np.ascontiguousarray(np.asarray(seq_lens), dtype=np.int32).reshape(-1)
    code = DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    rc = _lib.pa_decode_partition_for(lens.ctypes.data if lens.size else None, lens.size,
                                      num_kv_heads, head_dim, block_size, code, slots)
    if rc < 0:
        raise PagedAttnError(rc, "pa_decode_partition_for")
    return rc


def cached_workspace(device: torch.device) -> Optional[torch.Tensor]:
    """The split-partial workspace pa_decode currently uses on ``device``
    (None before the first call).  A CUDA graph that captured a decode keeps
    a reference to it, so that a later, larger request, which replaces the
    cached buffer, cannot free the memory the graph writes to."""
    return _ws_cache.get((device.index or 0, 0))


def _workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    key = (device.index or 0, 0)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def pa_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_tables: torch.Tensor, seq_lens: torch.Tensor, scale: float,
              block_size: Optional[int] = None, num_kv_heads: Optional[int] = None,
              max_seq_len: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
              partition_size: int = 0, variant: int = 0, merge: int = 0,
              heads_per_cta: int = 0, seq_order: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out float32 [B, Hq, D] <- paged attention of q [B, Hq, D] over the caches.

    max_seq_len (a host bound on seq_lens) defaults to the table width times
    the block size.  The workspace for split partials is taken from a cached
    device buffer unless one is given.  variant: 0 automatic, 1 CUDA cores, 2
    tensor cores, 3 tensor cores with one KV head per warp (heads_per_cta
    heads per CTA, 0 = the library's choice).  merge: 0 the library's choice,
    1 the reduce kernel, 2 inside the main kernel (pa_decode_opt).  seq_order
    (int32 [B] on the device, a permutation): the order in which the grid
    takes the sequences, e.g. longest first (decode_order)."""
    NB, Hkv, bs, D = k_cache.shape
    if block_size is not None and block_size != bs:
        raise ValueError(f"block_size {block_size} != cache block size {bs}")
    if num_kv_heads is not None and num_kv_heads != Hkv:
        raise ValueError(f"num_kv_heads {num_kv_heads} != cache heads {Hkv}")
    B, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q/out shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [B, W] and seq_lens [B]")
    W = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = W * bs
    need = decode_workspace_size(B, Hq, D, max_seq_len, partition_size)
    if workspace is None and need:
        workspace = _workspace(q.device, need)
    ws_ptr = 0 if workspace is None else _dev(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    order = None
    if seq_order is not None:
        if seq_order.numel() != B:
            raise ValueError("seq_order must have one entry per sequence")
        order = _dev(seq_order, "seq_order", torch.int32)
    opts = pa_decode_opts(int(partition_size), int(variant), int(merge), int(heads_per_cta),
                          order)
    _check(_lib.pa_decode_opt(
        _dev(out, "out", torch.float32), _dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache", k_cache.dtype), _dev(block_tables, "block_tables", torch.int32),
        _dev(seq_lens, "seq_lens", torch.int32), B, Hq, Hkv, D, bs, W, NB, int(max_seq_len),
        float(scale), DTYPE_CODE[k_cache.dtype], ws_ptr, ws_bytes, ctypes.byref(opts),
        _stream(q)), "pa_decode")
    return out


def pa_append_decode(out: torch.Tensor, q: torch.Tensor, k_new: torch.Tensor,
                     v_new: torch.Tensor, slot_mapping: torch.Tensor, k_cache: torch.Tensor,
                     v_cache: torch.Tensor, block_tables: torch.Tensor, seq_lens: torch.Tensor,
                     scale: float, max_seq_len: Optional[int] = None,
                     workspace: Optional[torch.Tensor] = None, partition_size: int = 0,
                     variant: int = 0, merge: int = 0, heads_per_cta: int = 0,
                     seq_order: Optional[torch.Tensor] = None) -> torch.Tensor:
    """pa_append_decode: each sequence's new token (k_new, v_new [B, Hkv, D]
    at slot_mapping[B], position seq_lens - 1) written into the caches and
    the decode over seq_lens tokens, in one launch (plus the reduce)."""
    NB, Hkv, bs, D = k_cache.shape
    B, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q/out shape mismatch")
    if tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D):
        raise ValueError(f"k_new/v_new must be [{B}, {Hkv}, {D}]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B or \
            slot_mapping.numel() != B:
        raise ValueError("block_tables [B, W], seq_lens [B], slot_mapping [B]")
    W = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = W * bs
    need = decode_workspace_size(B, Hq, D, max_seq_len, partition_size)
    if workspace is None and need:
        workspace = _workspace(q.device, need)
    ws_ptr = 0 if workspace is None else _dev(workspace, "workspace")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    order = None
    if seq_order is not None:
        if seq_order.numel() != B:
            raise ValueError("seq_order must have one entry per sequence")
        order = _dev(seq_order, "seq_order", torch.int32)
    opts = pa_decode_opts(int(partition_size), int(variant), int(merge), int(heads_per_cta),
                          order)
    dt = k_cache.dtype
    _check(_lib.pa_append_decode(
        _dev(out, "out", torch.float32), _dev(q, "q", dt), _dev(k_new, "k_new", dt),
        _dev(v_new, "v_new", dt), _dev(slot_mapping, "slot_mapping", torch.int64),
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", dt),
        _dev(block_tables, "block_tables", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        B, Hq, Hkv, D, bs, W, NB, int(max_seq_len), float(scale), DTYPE_CODE[dt], ws_ptr,
        ws_bytes, ctypes.byref(opts), _stream(q)), "pa_append_decode")
    return out


def pa_prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
               block_tables: torch.Tensor, seq_lens: torch.Tensor, cu_q_lens: torch.Tensor,
               scale: float, max_q_len: int, max_seq_len: Optional[int] = None,
               variant: int = 0) -> torch.Tensor:
    """Causal attention of each sequence's last n_s tokens (rows cu_q_lens[s]..
    cu_q_lens[s+1] of q [total, Hq, D]) over its paged context; out float32.
    variant: 0 automatic, 1 the mma.sync kernel, 2 the tcgen05 kernel, 3 the tcgen05
    kernel persistent (one CTA per SM over a share of the tiles), 4 the tcgen05
    kernel with P as one fp16 per weight (half the P.V products; each weight
    within 2^-11 instead of 2^-14; a bf16 V value beyond the fp16 range sets
    the "range" device error)."""
    NB, Hkv, bs, D = k_cache.shape
    total, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (total, Hq, D):
        raise ValueError("q/out shape mismatch")
    B = seq_lens.numel()
    if block_tables.dim() != 2 or block_tables.shape[0] != B or cu_q_lens.numel() != B + 1:
        raise ValueError("block_tables [B, W], seq_lens [B], cu_q_lens [B + 1]")
    W = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = W * bs
    _check(_lib.pa_prefill_ex(
        _dev(out, "out", torch.float32), _dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache", k_cache.dtype), _dev(block_tables, "block_tables", torch.int32),
        _dev(seq_lens, "seq_lens", torch.int32), _dev(cu_q_lens, "cu_q_lens", torch.int32), B, Hq,
        Hkv, D, bs, W, NB, int(max_q_len), int(max_seq_len), float(scale),
        DTYPE_CODE[k_cache.dtype], int(variant), _stream(q)), "pa_prefill")
    return out


def selftest_wait(limit_s: float, abort_after_s: float = 0.0) -> float:
    """Run the bounded-wait self-test on the current device and stream;
    returns the seconds the wait took (it sets the "timeout" device error)."""
    el = torch.zeros(1, dtype=torch.int64, device="cuda")
    _check(_lib.pa_selftest_wait(int(limit_s * 1e9), int(abort_after_s * 1e9), el.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream), "pa_selftest_wait")
    torch.cuda.synchronize()
    return int(el.item()) / 1e9


def pa_decode_static(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                     v_cache: torch.Tensor, block_tables: torch.Tensor, seq_lens: torch.Tensor,
                     scale: float, max_seq_len: Optional[int] = None) -> torch.Tensor:
    """pa_decode without a workspace, for callers that cannot allocate device
    memory: the split partials live in the library's fixed 32 MiB device
    array (shared by all calls; serialise calls that could overlap)."""
    NB, Hkv, bs, D = k_cache.shape
    B, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q/out shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [B, W] and seq_lens [B]")
    W = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = W * bs
    _check(_lib.pa_decode_static(
        _dev(out, "out", torch.float32), _dev(q, "q", k_cache.dtype), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache", k_cache.dtype), _dev(block_tables, "block_tables", torch.int32),
        _dev(seq_lens, "seq_lens", torch.int32), B, Hq, Hkv, D, bs, W, NB, int(max_seq_len),
        float(scale), DTYPE_CODE[k_cache.dtype], _stream(q)), "pa_decode_static")
    return out


def pa_copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, src_dst_pairs: torch.Tensor) -> None:
    """src_dst_pairs int64 [n, 2] on the device."""
    NB, Hkv, bs, D = k_cache.shape
    n = src_dst_pairs.shape[0] if src_dst_pairs.numel() else 0
    if n == 0:
        return
    block_bytes = Hkv * bs * D * k_cache.element_size()
    _check(_lib.pa_copy_blocks(
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", k_cache.dtype),
        _dev(src_dst_pairs, "src_dst_pairs", torch.int64), n, block_bytes, NB,
        _stream(k_cache)), "pa_copy_blocks")


def pa_swap_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                   src_v: torch.Tensor, src_dst_pairs: torch.Tensor) -> None:
    """Copy blocks between two caches of one block shape; a side may be pinned
    host memory (``tensor.pin_memory()``).  src_dst_pairs int64 [n, 2], on the
    device or pinned."""
    n = src_dst_pairs.shape[0] if src_dst_pairs.numel() else 0
    if n == 0:
        return
    if tuple(dst_k.shape[1:]) != tuple(src_k.shape[1:]) or dst_k.dtype != src_k.dtype:
        raise ValueError("caches differ in block shape or dtype")
    for name, t in (("dst_k", dst_k), ("dst_v", dst_v), ("src_k", src_k), ("src_v", src_v),
                    ("src_dst_pairs", src_dst_pairs)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if not (t.is_cuda or t.is_pinned()):
            raise TypeError(f"{name} must be a CUDA tensor or pinned host memory")
    if src_dst_pairs.dtype != torch.int64:
        raise TypeError("src_dst_pairs must be int64")
    NBd, Hkv, bs, D = dst_k.shape
    block_bytes = Hkv * bs * D * dst_k.element_size()
    dev = dst_k.device if dst_k.is_cuda else src_k.device
    _check(_lib.pa_swap_blocks(dst_k.data_ptr(), dst_v.data_ptr(), src_k.data_ptr(),
                               src_v.data_ptr(), src_dst_pairs.data_ptr(), n, block_bytes,
                               src_k.shape[0], NBd, torch.cuda.current_stream(dev).cuda_stream),
           "pa_swap_blocks")


# ----------------------------------------------------------------- allocator
def _np_ptr(a: np.ndarray) -> int:
    return a.ctypes.data


class BlockAllocator:
    """Handle on the C++ host allocator (pa_alloc_*, pa_seq_*)."""

    @classmethod
    def view(cls, handle: int, num_blocks: int, block_size: int) -> "BlockAllocator":
        """A handle on an allocator someone else owns (a pa_runtime's)."""
        self = cls.__new__(cls)
        self._h = ctypes.c_void_p(handle)
        self._owned = False
        self.num_blocks, self.block_size = num_blocks, block_size
        return self

    def __init__(self, num_blocks: int, block_size: int,
                 free_order: Optional[Sequence[int]] = None, max_blocks_per_seq: int = 0):
        self._owned = True
        self._h = ctypes.c_void_p()
        fo = None
        if free_order is not None:
            fo = np.ascontiguousarray(free_order, dtype=np.int32)
            if fo.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
        _check(_lib.pa_alloc_create(ctypes.byref(self._h), num_blocks, block_size,
                                    max_blocks_per_seq, None if fo is None else _np_ptr(fo)),
               "pa_alloc_create")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def __del__(self, _destroy=_lib.pa_alloc_destroy, _null=ctypes.c_void_p):
        # bound at definition time: at interpreter shutdown the module globals
        # (ctypes among them) may already be None
        h = getattr(self, "_h", None)
        if h is not None and h.value and getattr(self, "_owned", True):
            _destroy(h)
            self._h = _null()

    def seq_add(self, seq_id: int) -> None:
        _check(_lib.pa_seq_add(self._h, seq_id), "pa_seq_add")

    def seq_append(self, seq_id: int, n: int) -> Tuple[np.ndarray, Optional[Tuple[int, int]]]:
        slots = np.empty(max(n, 1), np.int64)
        pair = np.empty(2, np.int64)
        ncow = ctypes.c_int(0)
        _check(_lib.pa_seq_append(self._h, seq_id, n, _np_ptr(slots), _np_ptr(pair),
                                  ctypes.addressof(ncow)), "pa_seq_append")
        return slots[:n], ((int(pair[0]), int(pair[1])) if ncow.value else None)

    def batch_append(self, seq_ids: Sequence[int], n_tokens: Optional[Sequence[int]] = None,
                     slots_out: Optional[np.ndarray] = None
                     ) -> Tuple[np.ndarray, np.ndarray]:
        """Returns (slots int64 [sum n], cow pairs int64 [k, 2])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        nt = None if n_tokens is None else np.ascontiguousarray(n_tokens, dtype=np.int32)
        total = ids.shape[0] if nt is None else int(nt.sum())
        slots = slots_out if slots_out is not None else np.empty(max(total, 1), np.int64)
        pairs = np.empty((max(ids.shape[0], 1), 2), np.int64)
        ncow = ctypes.c_int(0)
        _check(_lib.pa_batch_append(self._h, _np_ptr(ids), ids.shape[0],
                                    None if nt is None else _np_ptr(nt), _np_ptr(slots),
                                    _np_ptr(pairs), ctypes.addressof(ncow)), "pa_batch_append")
        return slots[:total], pairs[:ncow.value]

    def step_layout(self, events: np.ndarray, num_seqs: int, width: int) -> pa_step_layout:
        """pa_step_plan's layout for these events, without applying them."""
        ev = np.ascontiguousarray(events, dtype=np.int64).reshape(-1, 3)
        lay = pa_step_layout()
        ids = np.zeros(max(num_seqs, 1), np.int64)
        _check(_lib.pa_step_plan(self._h, _np_ptr(ev), ev.shape[0], _np_ptr(ids), num_seqs,
                                 width, None, 0, None, ctypes.byref(lay)), "pa_step_plan")
        return lay

    def step_plan(self, events: np.ndarray, decode_ids: np.ndarray, width: int,
                  stage: np.ndarray, pairs_before: Optional[np.ndarray] = None
                  ) -> pa_step_layout:
        """Applies a step's events (int64 [n, 3]) and writes slots, copy pairs,
        table rows and lengths into ``stage`` (a uint8 array, e.g. a view of
        page-locked memory) at the returned layout's offsets; ``pairs_before``
        (int32 [n + 1]) receives the pair count before each event."""
        ev = np.ascontiguousarray(events, dtype=np.int64).reshape(-1, 3)
        ids = np.ascontiguousarray(decode_ids, dtype=np.int64)
        lay = pa_step_layout()
        rc = _lib.pa_step_plan(self._h, _np_ptr(ev), ev.shape[0],
                               _np_ptr(ids) if ids.size else None, ids.size, width,
                               stage.ctypes.data, stage.nbytes,
                               None if pairs_before is None else _np_ptr(pairs_before),
                               ctypes.byref(lay))
        if rc != 0:
            err = PagedAttnError(rc, "pa_step_plan")
            err.layout = lay  # events_applied: where the step stopped
            raise err
        return lay

    def seq_fork(self, parent: int, child: int) -> None:
        _check(_lib.pa_seq_fork(self._h, parent, child), "pa_seq_fork")

    def seq_free(self, seq_id: int) -> None:
        _check(_lib.pa_seq_free(self._h, seq_id), "pa_seq_free")

    def seq_block_table(self, seq_id: int) -> Tuple[List[int], int]:
        n = ctypes.c_int(0)
        L = ctypes.c_int64(0)
        _check(_lib.pa_seq_block_table(self._h, seq_id, None, 0, ctypes.addressof(n),
                                       ctypes.addressof(L)), "pa_seq_block_table")
        buf = np.empty(max(n.value, 1), np.int32)
        _check(_lib.pa_seq_block_table(self._h, seq_id, _np_ptr(buf), n.value, None, None),
               "pa_seq_block_table")
        return buf[:n.value].tolist(), L.value

    def block_tables(self, seq_ids: Sequence[int], width: int,
                     tables_out: Optional[np.ndarray] = None,
                     lens_out: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = tables_out if tables_out is not None else np.empty((ids.shape[0], width), np.int32)
        lens = lens_out if lens_out is not None else np.empty(ids.shape[0], np.int32)
        _check(_lib.pa_block_tables(self._h, _np_ptr(ids), ids.shape[0], _np_ptr(tables), width,
                                    _np_ptr(lens)), "pa_block_tables")
        return tables, lens

    def stats(self) -> dict:
        st = pa_alloc_stats_t()
        _check(_lib.pa_alloc_stats(self._h, ctypes.byref(st)), "pa_alloc_stats")
        return {n: getattr(st, n) for n, _ in pa_alloc_stats_t._fields_}

    def free_list(self) -> List[int]:
        n = ctypes.c_int(0)
        _check(_lib.pa_alloc_free_list(self._h, None, 0, ctypes.addressof(n)), "pa_alloc_free_list")
        buf = np.empty(max(n.value, 1), np.int32)
        _check(_lib.pa_alloc_free_list(self._h, _np_ptr(buf), n.value, None), "pa_alloc_free_list")
        return buf[:n.value].tolist()

    def refcount(self, block: int) -> int:
        return _lib.pa_alloc_refcount(self._h, block)

    # prefix caching
    def seq_add_cached(self, seq_id: int, token_ids: Sequence[int]) -> int:
        """New sequence sharing the longest indexed prefix; returns the number
        of cached tokens (a multiple of the block size)."""
        t = np.ascontiguousarray(token_ids, dtype=np.int64)
        n = ctypes.c_int(0)
        _check(_lib.pa_seq_add_cached(self._h, seq_id, _np_ptr(t) if t.size else None, t.size,
                                      ctypes.addressof(n)), "pa_seq_add_cached")
        return n.value

    def seq_append_tokens(self, seq_id: int, token_ids: Sequence[int]
                          ) -> Tuple[np.ndarray, Optional[Tuple[int, int]]]:
        t = np.ascontiguousarray(token_ids, dtype=np.int64)
        slots = np.empty(max(t.size, 1), np.int64)
        pair = np.empty(2, np.int64)
        ncow = ctypes.c_int(0)
        _check(_lib.pa_seq_append_tokens(self._h, seq_id, _np_ptr(t) if t.size else None, t.size,
                                         _np_ptr(slots), _np_ptr(pair), ctypes.addressof(ncow)),
               "pa_seq_append_tokens")
        return slots[:t.size], ((int(pair[0]), int(pair[1])) if ncow.value else None)

    # swap
    def set_host_pool(self, num_host_blocks: int) -> None:
        _check(_lib.pa_alloc_set_host_pool(self._h, num_host_blocks), "pa_alloc_set_host_pool")

    def _swap(self, fn, name, seq_id: int) -> np.ndarray:
        n = ctypes.c_int(0)
        cap = max(self.num_blocks, 1)
        pairs = np.empty((cap, 2), np.int64)
        _check(fn(self._h, seq_id, _np_ptr(pairs), cap, ctypes.addressof(n)), name)
        return pairs[:n.value].copy()

    def seq_swap_out(self, seq_id: int) -> np.ndarray:
        """(device block, host block) pairs, in logical order."""
        return self._swap(_lib.pa_seq_swap_out, "pa_seq_swap_out", seq_id)

    def seq_swap_in(self, seq_id: int) -> np.ndarray:
        """(host block, device block) pairs, in logical order."""
        return self._swap(_lib.pa_seq_swap_in, "pa_seq_swap_in", seq_id)


# ----------------------------------------------------------------- runtime
class Runtime:
    """pa_runtime: one C call per host-fed decode step over caller-owned
    caches (see pagedattn.h, "Runtime").  Host tensors passed to step()
    should be page-locked; the step's output is in ``out`` once the returned
    event has completed (wait_event)."""

    def __init__(self, k_cache: torch.Tensor, v_cache: torch.Tensor, num_heads: int,
                 table_width: int, max_batch: int, max_new_tokens: int, scale: float,
                 free_order: Optional[Sequence[int]] = None, max_blocks_per_seq: int = 0):
        NB, Hkv, bs, D = k_cache.shape
        self.k_cache, self.v_cache = k_cache, v_cache   # kept alive with the runtime
        self.cfg = pa_runtime_config(NB, bs, num_heads, Hkv, D, DTYPE_CODE[k_cache.dtype],
                                     table_width, max_batch, max_new_tokens, max_blocks_per_seq,
                                     scale)
        fo = None
        if free_order is not None:
            fo = np.ascontiguousarray(free_order, dtype=np.int32)
        self._h = ctypes.c_void_p()
        _check(_lib.pa_rt_create(ctypes.byref(self._h), ctypes.byref(self.cfg),
                                 _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache", k_cache.dtype),
                                 None if fo is None else _np_ptr(fo)), "pa_rt_create")
        self.alloc = BlockAllocator.view(_lib.pa_rt_allocator(self._h), NB, bs)
        self._ready = ctypes.c_void_p()

    def __del__(self, _destroy=_lib.pa_rt_destroy, _null=ctypes.c_void_p):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            _destroy(h)
            self._h = _null()

    def step(self, events: np.ndarray, decode_ids: np.ndarray, k_new: Optional[torch.Tensor],
             v_new: Optional[torch.Tensor], q: Optional[torch.Tensor],
             out: Optional[torch.Tensor]) -> int:
        """One step; returns its "ready" event (a cudaEvent_t as an int)."""
        rc = _lib.pa_rt_step(self._h, events.ctypes.data, events.shape[0],
                             decode_ids.ctypes.data if decode_ids.size else None, decode_ids.size,
                             None if k_new is None else k_new.data_ptr(),
                             None if v_new is None else v_new.data_ptr(),
                             None if q is None else q.data_ptr(),
                             None if out is None else out.data_ptr(), ctypes.byref(self._ready))
        if rc != 0:
            raise PagedAttnError(rc, "pa_rt_step")
        return self._ready.value

    @staticmethod
    def wait_event(event: int) -> None:
        _check(_lib.pa_event_wait(event), "pa_event_wait")

    def wait(self) -> None:
        _check(_lib.pa_rt_wait(self._h), "pa_rt_wait")

    def stats(self) -> dict:
        v = [ctypes.c_int64() for _ in range(3)]
        _check(_lib.pa_rt_stats(self._h, *(ctypes.addressof(x) for x in v)), "pa_rt_stats")
        return {"steps": v[0].value, "replays": v[1].value, "captures": v[2].value}
