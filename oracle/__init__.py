"""fp64 CPU oracles: paged decode attention (paged_decode_oracle.c) and the decode
projection GEMV (gemv_oracle.c), through ctypes.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` import this package.  The CUDA library
(``decode_attention_paged_split_b200``) does not import it and shares no code
with it.

Every function takes a ``workloads.Workload``-like object (torch CPU tensors:
bf16 q / k_cache / v_cache, int32 page_table / seq_lens) and returns float64
numpy arrays.  What is computed, and the readings taken where the source pages
are silent, is documented at the top of ``paged_decode_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

_lib = None


class _Problem(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p),
        ("q_stride", ctypes.c_int64 * 3),
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("kv_stride", ctypes.c_int64 * 4),
        ("page_table", ctypes.c_void_p),
        ("pt_stride", ctypes.c_int64 * 2),
        ("seq_lens", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("scale", ctypes.c_double),
    ]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER(_Problem)
        dp = ctypes.POINTER(ctypes.c_double)
        L.oracle_paged_decode.argtypes = [P, dp, ctypes.c_int]
        L.oracle_paged_decode_rows.argtypes = [P, ctypes.c_void_p, ctypes.c_int64, dp, ctypes.c_int]
        L.oracle_paged_decode_split.argtypes = [P, ctypes.c_int, dp, ctypes.c_int]
        L.oracle_paged_decode_chunks.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, dp]
        L.oracle_partial.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, dp, dp, dp]
        L.oracle_round_bf16.argtypes = [ctypes.c_double]
        L.oracle_round_bf16.restype = ctypes.c_uint16
        L.oracle_round_bf16_array.argtypes = [dp, ctypes.c_int64, ctypes.c_void_p]
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


class _Bound:
    """Keeps the host tensors alive while the C struct points into them."""

    def __init__(self, w):
        q, k, v = w.q, w.k_cache, w.v_cache
        pt = w.page_table.to(torch.int32)
        sl = w.seq_lens.to(torch.int32).contiguous()
        for t in (q, k, v):
            assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
        assert k.shape == v.shape and k.stride() == v.stride()
        self.keep = (q, k, v, pt, sl)
        s = _Problem()
        s.q = q.data_ptr()
        s.q_stride = (ctypes.c_int64 * 3)(*q.stride())
        s.k = k.data_ptr()
        s.v = v.data_ptr()
        s.kv_stride = (ctypes.c_int64 * 4)(*k.stride())
        s.page_table = pt.data_ptr()
        s.pt_stride = (ctypes.c_int64 * 2)(*pt.stride())
        s.seq_lens = sl.data_ptr()
        s.batch = q.shape[0]
        s.num_q_heads = q.shape[1]
        s.num_kv_heads = k.shape[2]
        s.head_dim = q.shape[2]
        s.page_size = k.shape[1]
        s.num_pages = k.shape[0]
        s.max_pages = pt.shape[1]
        s.scale = float(w.scale)
        self.s = s


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def paged_decode(w, nthreads: int = 0) -> np.ndarray:
    """The definition for every (b, h): float64 [B, Hq, D]."""
    bnd = _Bound(w)
    out = np.zeros((w.q.shape[0], w.q.shape[1], w.q.shape[2]), dtype=np.float64)
    _check(lib().oracle_paged_decode(ctypes.byref(bnd.s), _dptr(out), nthreads), "paged_decode")
    return out


def paged_decode_rows(w, rows, nthreads: int = 0) -> np.ndarray:
    """The definition for the listed (b, h) rows only: float64 [len(rows), D]."""
    bnd = _Bound(w)
    bh = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 2))
    out = np.zeros((bh.shape[0], w.q.shape[2]), dtype=np.float64)
    _check(lib().oracle_paged_decode_rows(ctypes.byref(bnd.s), bh.ctypes.data, bh.shape[0], _dptr(out), nthreads),
           "paged_decode_rows")
    return out


def paged_decode_split(w, num_splits: int, nthreads: int = 0) -> np.ndarray:
    """Split form (page-aligned min(S, n_b) chunks, then combine): float64 [B, Hq, D]."""
    bnd = _Bound(w)
    out = np.zeros((w.q.shape[0], w.q.shape[1], w.q.shape[2]), dtype=np.float64)
    _check(lib().oracle_paged_decode_split(ctypes.byref(bnd.s), num_splits, _dptr(out), nthreads), "split")
    return out


def paged_decode_chunks(w, b: int, h: int, bounds) -> np.ndarray:
    """Split form over explicit token boundaries [0, ..., L_b] for one (b, h)."""
    bnd = _Bound(w)
    bo = np.ascontiguousarray(np.asarray(bounds, dtype=np.int64))
    out = np.zeros(w.q.shape[2], dtype=np.float64)
    _check(lib().oracle_paged_decode_chunks(ctypes.byref(bnd.s), b, h, bo.ctypes.data, bo.shape[0], _dptr(out)),
           "chunks")
    return out


def partial(w, b: int, h: int, t0: int, t1: int):
    """(acc[D], m, l) over tokens [t0, t1) of (b, h), all float64."""
    bnd = _Bound(w)
    acc = np.zeros(w.q.shape[2], dtype=np.float64)
    m = ctypes.c_double()
    l = ctypes.c_double()
    _check(lib().oracle_partial(ctypes.byref(bnd.s), b, h, t0, t1, _dptr(acc), ctypes.byref(m), ctypes.byref(l)),
           "partial")
    return acc, m.value, l.value


def round_bf16(x) -> torch.Tensor:
    """Round float64 values to bf16 (nearest, ties to even); returns a torch bf16 tensor."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    bits = np.zeros(a.shape, dtype=np.uint16)
    lib().oracle_round_bf16_array(_dptr(a), a.size, bits.ctypes.data)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def num_host_cores() -> int:
    return os.cpu_count() or 1


_gemv_lib = None


def _gemv():
    global _gemv_lib
    if _gemv_lib is None:
        L = ctypes.CDLL(_build.build_gemv())
        dp = ctypes.POINTER(ctypes.c_double)
        L.oracle_gemv.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_int, dp, dp, ctypes.c_int]
        _gemv_lib = L
    return _gemv_lib


def gemv(x: torch.Tensor, w: torch.Tensor, nthreads: int = 0):
    """y = x W^T in fp64 for bf16 x [M, K] and W [N, K] (rows contiguous); returns
    (y, absy), both float64 [M, N], absy[m, n] = sum_k |x[m, k] W[n, k]|."""
    assert x.dtype == torch.bfloat16 and w.dtype == torch.bfloat16 and x.device.type == "cpu"
    assert x.stride(1) == 1 and w.stride(1) == 1 and x.shape[1] == w.shape[1]
    M, K = x.shape
    N = w.shape[0]
    y = np.zeros((M, N), dtype=np.float64)
    a = np.zeros((M, N), dtype=np.float64)
    _check(_gemv().oracle_gemv(x.data_ptr(), x.stride(0), w.data_ptr(), w.stride(0), M, N, K, _dptr(y), _dptr(a),
                               nthreads), "gemv")
    return y, a


class _PrefillProblem(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p),
        ("q_stride", ctypes.c_int64 * 4),
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("kv_stride", ctypes.c_int64 * 4),
        ("page_table", ctypes.c_void_p),
        ("pt_stride", ctypes.c_int64 * 2),
        ("seq_lens", ctypes.c_void_p),
        ("mask", ctypes.c_void_p),
        ("mask_stride", ctypes.c_int64 * 3),
        ("mask_kv_len", ctypes.c_int64),
        ("batch", ctypes.c_int32),
        ("q_len", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("causal_offset", ctypes.c_int32),
        ("scale", ctypes.c_double),
    ]


_prefill_lib = None


def _prefill():
    global _prefill_lib
    if _prefill_lib is None:
        L = ctypes.CDLL(_build.build_prefill())
        L.oracle_paged_prefill.argtypes = [ctypes.POINTER(_PrefillProblem), ctypes.POINTER(ctypes.c_double),
                                           ctypes.c_int]
        _prefill_lib = L
    return _prefill_lib


def paged_prefill(w, nthreads: int = 0) -> np.ndarray:
    """Multi-query attention of a ``workloads.PrefillWorkload``: float64 [B, Lq, Hq, D]."""
    q, k, v = w.q, w.k_cache, w.v_cache
    pt = w.page_table.to(torch.int32)
    sl = w.seq_lens.to(torch.int32).contiguous()
    mask = w.mask
    keep = [q, k, v, pt, sl, mask]
    s = _PrefillProblem()
    s.q = q.data_ptr()
    s.q_stride = (ctypes.c_int64 * 4)(*q.stride())
    s.k, s.v = k.data_ptr(), v.data_ptr()
    s.kv_stride = (ctypes.c_int64 * 4)(*k.stride())
    s.page_table = pt.data_ptr()
    s.pt_stride = (ctypes.c_int64 * 2)(*pt.stride())
    s.seq_lens = sl.data_ptr()
    if mask is not None:
        assert mask.dtype == torch.uint8
        ms = mask.stride()
        s.mask = mask.data_ptr()
        s.mask_stride = (ctypes.c_int64 * 3)(ms[0], 0, ms[1]) if mask.dim() == 2 else (ctypes.c_int64 * 3)(*ms)
        s.mask_kv_len = mask.shape[-1]
    s.batch, s.q_len, s.num_q_heads, s.head_dim = q.shape[0], q.shape[1], q.shape[2], q.shape[3]
    s.num_kv_heads, s.page_size, s.num_pages, s.max_pages = k.shape[2], k.shape[1], k.shape[0], pt.shape[1]
    s.causal_offset = int(w.causal_offset)
    s.scale = float(w.scale)
    out = np.zeros(tuple(q.shape), dtype=np.float64)
    _check(_prefill().oracle_paged_prefill(ctypes.byref(s), _dptr(out), nthreads), "paged_prefill")
    del keep
    return out
