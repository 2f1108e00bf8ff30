"""Oracle attention -- TEST INFRASTRUCTURE ONLY (see oracle/__init__).

* ``paged_decode``  -- ctypes entry to the fp64 C loop in attn_ref.c, which
  gathers every token through the block table (mbrenndoerfer.com "Paged
  Attention > Summary", bullet 3) and applies the exact two-pass softmax;
* ``contiguous_attention`` -- numpy fp64 brute force of softmax(q K^T s) V over
  K/V that are already in logical order; the statement that paging does not
  change the attention result (paweldubiel.com "PagedAttention", first section
  and "Text order is not a memory address") makes this the same quantity;
* ``gather_logical`` -- numpy gather of a sequence's K/V through its table;
* ``partial_state`` / ``merge_partials`` -- the split-context decomposition
  of the same softmax: a token range r gives (m_r, l_r, o_r) with
  m_r = max x_t, l_r = sum exp(x_t - m_r), o_r = sum exp(x_t - m_r) v_t; the
  ranges combine as out = sum_r e^(m_r - M) o_r / sum_r e^(m_r - M) l_r with
  M = max_r m_r.  This is the online-softmax merge that mbrenndoerfer.com's
  bullet 3 names for block-at-a-time processing, applied to whole ranges;
* ``decode_storage`` -- stored bytes to float64 (f32, bf16, f16).
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

from . import build as _build

_DT = {"f32": 0, "bf16": 1, "f16": 2}
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.attn_ref_decode.restype = ctypes.c_int
        L.attn_ref_decode.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
        L.attn_ref_decode_value.restype = ctypes.c_double
        L.attn_ref_decode_value.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_longlong]
        L.attn_ref_max_threads.restype = ctypes.c_int
        L.attn_ref_prefill.restype = ctypes.c_int
        L.attn_ref_prefill.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, ctypes.c_int]
        L.attn_ref_prefill_sel.restype = ctypes.c_int
        L.attn_ref_prefill_sel.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
        _lib = L
    return _lib


def max_threads() -> int:
    return lib().attn_ref_max_threads()


def _dtype_name(t: torch.Tensor) -> str:
    return {torch.float32: "f32", torch.bfloat16: "bf16", torch.float16: "f16"}[t.dtype]


def paged_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 block_tables: np.ndarray, seq_lens: np.ndarray, scale: float,
                 sel: Optional[Sequence[Tuple[int, int]]] = None, n_threads: int = 0) -> np.ndarray:
    """fp64 attention over the paged cache.

    q [B, Hq, D] and the caches [NB, Hkv, bs, D] are CPU tensors in their
    storage dtype; block_tables int32 [B, max_blocks]; seq_lens int32 [B].
    Returns float64 [B, Hq, D], or [len(sel), D] for a list of (s, h) pairs.
    """
    assert q.device.type == "cpu" and k_cache.device.type == "cpu"
    assert q.dtype == k_cache.dtype == v_cache.dtype
    q = q.contiguous(); k_cache = k_cache.contiguous(); v_cache = v_cache.contiguous()
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    assert D2 == D and tuple(v_cache.shape) == tuple(k_cache.shape)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    if bt.ndim == 1:
        bt = bt.reshape(B, -1)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert bt.shape[0] == B and sl.shape == (B,)
    max_blocks = bt.shape[1]
    if sel is None:
        out = np.zeros((B, Hq, D), np.float64)
        sel_arr, n_sel = None, 0
    else:
        sel_arr = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(-1, 2))
        n_sel = sel_arr.shape[0]
        out = np.zeros((n_sel, D), np.float64)
    rc = lib().attn_ref_decode(
        out.ctypes.data, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        _DT[_dtype_name(q)], bt.ctypes.data, sl.ctypes.data, B, Hq, Hkv, D, bs,
        max_blocks, NB, float(scale), None if sel_arr is None else sel_arr.ctypes.data,
        n_sel, int(n_threads))
    if rc != 0:
        raise ValueError("oracle: bad argument or block-table entry out of range")
    return out


def paged_prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  block_tables: np.ndarray, seq_lens: np.ndarray, cu_q: np.ndarray,
                  scale: float, n_threads: int = 0,
                  sel: Optional[Sequence[Tuple[int, int]]] = None) -> np.ndarray:
    """fp64 causal attention of chunk rows over the paged cache.

    q [total, Hq, D] holds, for sequence s, rows cu_q[s]..cu_q[s+1]-1 at
    positions L_s - n_s .. L_s - 1 (n_s = cu_q[s+1] - cu_q[s]); each attends to
    tokens 0..its position.  Returns float64 [total, Hq, D], or [len(sel), D]
    for a list of (row, head) pairs."""
    q = q.contiguous(); k_cache = k_cache.contiguous(); v_cache = v_cache.contiguous()
    total, Hq, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    cu = np.ascontiguousarray(cu_q, dtype=np.int32)
    B = sl.shape[0]
    assert cu.shape == (B + 1,) and int(cu[-1]) == total and bt.shape[0] == B
    if sel is not None:
        sa = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(-1, 2))
        out = np.zeros((sa.shape[0], D), np.float64)
        rc = lib().attn_ref_prefill_sel(out.ctypes.data, q.data_ptr(), k_cache.data_ptr(),
                                        v_cache.data_ptr(), _DT[_dtype_name(q)], bt.ctypes.data,
                                        sl.ctypes.data, cu.ctypes.data, B, Hq, Hkv, D, bs,
                                        bt.shape[1], NB, float(scale), sa.ctypes.data,
                                        sa.shape[0], int(n_threads))
        if rc != 0:
            raise ValueError("oracle: bad prefill argument or table entry out of range")
        return out
    out = np.zeros((total, Hq, D), np.float64)
    rc = lib().attn_ref_prefill(out.ctypes.data, q.data_ptr(), k_cache.data_ptr(),
                                v_cache.data_ptr(), _DT[_dtype_name(q)], bt.ctypes.data,
                                sl.ctypes.data, cu.ctypes.data, B, Hq, Hkv, D, bs, bt.shape[1],
                                NB, float(scale), int(n_threads))
    if rc != 0:
        raise ValueError("oracle: bad prefill argument or table entry out of range")
    return out


def decode_storage(t: torch.Tensor) -> np.ndarray:
    """Stored values as float64, by each format's definition: bf16 is the high
    half of a binary32; f16 and f32 are IEEE binary16 / binary32."""
    t = t.contiguous()
    if t.dtype == torch.float32:
        return t.numpy().astype(np.float64)
    if t.dtype == torch.float16:
        return t.view(torch.int16).numpy().view(np.float16).astype(np.float64)
    if t.dtype == torch.bfloat16:
        bits = t.view(torch.int16).numpy().view(np.uint16).astype(np.uint32) << 16
        with np.errstate(invalid="ignore"):  # NaN patterns stay NaN
            return bits.view(np.float32).astype(np.float64)
    raise TypeError(t.dtype)


def contiguous_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(q K^T * scale) V in float64 for one query row q [D] over K, V [L, D]."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], np.float64)
    x = scale * (K @ q)
    w = np.exp(x - x.max())
    return (w @ V) / w.sum()


def gather_logical(cache: np.ndarray, table: Sequence[int], length: int, kv_head: int) -> np.ndarray:
    """Rows 0..length-1 of one KV head of one sequence, in logical order, from a
    [NB, Hkv, bs, D] float64 cache."""
    bs = cache.shape[2]
    t = np.arange(length)
    pb = np.asarray(table, dtype=np.int64)[t // bs]
    return cache[pb, kv_head, t % bs, :]


def partial_state(x: np.ndarray, V: np.ndarray) -> Tuple[float, float, np.ndarray]:
    """(m, l, o) of one token range: logits x [n], values V [n, D]."""
    if x.shape[0] == 0:
        return -np.inf, 0.0, np.zeros(V.shape[1], np.float64)
    m = float(x.max())
    w = np.exp(x - m)
    return m, float(w.sum()), w @ V


def merge_partials(states: List[Tuple[float, float, np.ndarray]]) -> np.ndarray:
    """Combine per-range (m, l, o) into the normalised output."""
    M = max(s[0] for s in states)
    if M == -np.inf:
        return np.zeros_like(states[0][2])
    num = sum(np.exp(m - M) * o for m, _, o in states if m != -np.inf)
    den = sum(np.exp(m - M) * l for m, l, _ in states if m != -np.inf)
    return num / den
