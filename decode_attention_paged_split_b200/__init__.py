"""Python binding of libattn_paged_decode.so: paged split-KV decode attention on B200.

Argument marshalling only.  Every step of the computation runs in the library's
CUDA kernels; PyTorch supplies device memory and the current stream.  There is
no CPU fallback: if the library is missing or fails to load, every call raises.

The operation (AstrAI commit d565d44c, ``csrc/kernels/attn_paged_decode.cu``,
commit log): single-token decode attention over a paged bf16 KV cache with
grouped-query attention, split-KV partials (o_part / ml_part) and one combine
kernel.  The C declarations, with argument meaning, layout, ownership and error
behaviour, are in ``include/attn_paged_decode.h``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "APDError",
    "attn_paged_decode",
    "attn_contig_decode",
    "attn_paged_prefill",
    "selftest_bounded_wait",
    "selftest_shared_ring_release",
    "selftest_mq_tc_stall",
    "gemv",
    "gemv_workspace_size",
    "DecodeCall",
    "attn_paged_decode_noalloc",
    "NOALLOC_SCRATCH_BYTES",
    "workspace_size",
    "alloc_workspace",
    "workspace_init",
    "read_device_flags",
    "query_plan",
    "status_string",
    "library_path",
    "FLAG_PAGE_OUT_OF_RANGE",
    "FLAG_SEQ_LEN_CLAMPED",
    "FLAG_SEQ_LEN_NEGATIVE",
    "FLAG_WAIT_TIMEOUT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libattn_paged_decode.so")

DTYPE_BF16, DTYPE_INT32, DTYPE_FP32 = 1, 2, 3
FLAG_PAGE_OUT_OF_RANGE = 0x1
FLAG_SEQ_LEN_CLAMPED = 0x2
FLAG_SEQ_LEN_NEGATIVE = 0x4
FLAG_WAIT_TIMEOUT = 0x8
NOALLOC_SCRATCH_BYTES = 8 << 20  # APD_NOALLOC_SCRATCH_BYTES

DTYPE_UINT8 = 4
_DTYPES = {torch.bfloat16: DTYPE_BF16, torch.int32: DTYPE_INT32, torch.float32: DTYPE_FP32,
           torch.uint8: DTYPE_UINT8, torch.bool: DTYPE_UINT8}


class _Tensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("ndim", ctypes.c_int32),
        ("shape", ctypes.c_int64 * 4),
        ("stride", ctypes.c_int64 * 4),
    ]


class _Plan(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int32),
        ("num_workers", ctypes.c_int32),
        ("grid_ctas", ctypes.c_int32),
        ("warps_per_cta", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("rows_per_unit", ctypes.c_int32),
        ("head_blocks", ctypes.c_int32),
        ("combine_ctas", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int64),
        ("partial_slots", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_int64),
        ("shared_kv_ring", ctypes.c_int32),
        ("cluster_size", ctypes.c_int32),
        ("q_head_blocks", ctypes.c_int32),
        ("q_heads_per_block", ctypes.c_int32),
    ]


class _Options(ctypes.Structure):
    _fields_ = [
        ("split_done_event", ctypes.c_void_p),
        ("disable_pdl", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("host_seq_lens", ctypes.c_void_p),
    ]


def _host_lens(host_seq_lens, batch: int):
    """The host_seq_lens hint as a contiguous int32 CPU tensor of `batch` entries (kept
    alive by the caller for the duration of the call), or None."""
    if host_seq_lens is None:
        return None
    t = torch.as_tensor(host_seq_lens, dtype=torch.int32, device="cpu").contiguous()
    if t.dim() != 1 or t.numel() != batch:
        raise ValueError(f"host_seq_lens must hold {batch} lengths, got shape {tuple(t.shape)}")
    return t


class _GemvPlan(ctypes.Structure):
    _fields_ = [
        ("workers", ctypes.c_int32),
        ("grid_ctas", ctypes.c_int32),
        ("warps_per_cta", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("x_staged", ctypes.c_int32),
        ("sum_ctas", ctypes.c_int32),
        ("cta_per_mtile", ctypes.c_int32),
        ("workspace_bytes", ctypes.c_int64),
    ]


class APDError(RuntimeError):
    """A non-zero apd_status returned by the library."""

    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: status {status} ({status_string(status)})"
        if status == 11:  # APD_ERR_CUDA
            msg += f": {_load().apd_last_cuda_error().decode(errors='replace')}"
        super().__init__(msg)


_lib = None


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with `python -m decode_attention_paged_split_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(_LIB_PATH)
    T = ctypes.POINTER(_Tensor)
    L.apd_workspace_size.argtypes = [ctypes.c_int] * 5
    L.apd_workspace_size.restype = ctypes.c_size_t
    L.apd_workspace_init.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    L.apd_workspace_init.restype = ctypes.c_int
    L.apd_attn_paged_decode.argtypes = [T, T, T, T, T, T, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_size_t, ctypes.c_void_p]
    L.apd_attn_paged_decode.restype = ctypes.c_int
    L.apd_attn_paged_decode_ex.argtypes = L.apd_attn_paged_decode.argtypes + [ctypes.POINTER(_Options)]
    L.apd_attn_contig_decode.argtypes = [T, T, T, T, T, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]
    L.apd_attn_contig_decode.restype = ctypes.c_int
    L.apd_attn_contig_decode_ex.argtypes = L.apd_attn_contig_decode.argtypes + [ctypes.POINTER(_Options)]
    L.apd_attn_contig_decode_ex.restype = ctypes.c_int
    L.apd_attn_paged_decode_ex.restype = ctypes.c_int
    L.apd_attn_paged_decode_noalloc.argtypes = [T, T, T, T, T, T, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
    L.apd_attn_paged_decode_noalloc.restype = ctypes.c_int
    L.apd_attn_paged_prefill.argtypes = [T, T, T, T, T, T, T, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
    L.apd_attn_paged_prefill.restype = ctypes.c_int
    L.apd_attn_paged_prefill_ex.argtypes = [T, T, T, T, T, T, T, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_int]
    L.apd_attn_paged_prefill_ex.restype = ctypes.c_int
    L.apd_selftest_bounded_wait.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p]
    L.apd_selftest_bounded_wait.restype = ctypes.c_int
    L.apd_selftest_shared_ring_release.argtypes = [T, T, T, T, T, T, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t,
                                                   ctypes.c_uint64, ctypes.c_void_p]
    L.apd_selftest_shared_ring_release.restype = ctypes.c_int
    L.apd_selftest_mq_tc_stall.argtypes = [T, T, T, T, T, T, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_size_t, ctypes.c_uint64, ctypes.c_void_p]
    L.apd_selftest_mq_tc_stall.restype = ctypes.c_int
    L.apd_gemv_workspace_size.argtypes = [ctypes.c_int] * 3
    L.apd_gemv_workspace_size.restype = ctypes.c_size_t
    L.apd_gemv_query_plan.argtypes = [ctypes.c_int] * 4 + [ctypes.POINTER(_GemvPlan)]
    L.apd_gemv_query_plan.restype = ctypes.c_int
    L.apd_gemv_bf16.argtypes = [T, T, T, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    L.apd_gemv_bf16.restype = ctypes.c_int
    L.apd_read_device_flags.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                        ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
    L.apd_read_device_flags.restype = ctypes.c_int
    L.apd_query_plan.argtypes = [ctypes.c_int] * 5 + [ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(_Plan)]
    L.apd_query_plan.restype = ctypes.c_int
    L.apd_query_plan_ex.argtypes = [ctypes.c_int] * 5 + [ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p,
                                                         ctypes.c_int64, ctypes.POINTER(_Plan)]
    L.apd_query_plan_ex.restype = ctypes.c_int
    L.apd_status_string.argtypes = [ctypes.c_int]
    L.apd_status_string.restype = ctypes.c_char_p
    L.apd_last_cuda_error.argtypes = []
    L.apd_last_cuda_error.restype = ctypes.c_char_p
    _lib = L
    return L


def lib():
    """The loaded ctypes library (raises if it is missing)."""
    return _load()


def status_string(status: int) -> str:
    return _load().apd_status_string(int(status)).decode()


_I64x4 = ctypes.c_int64 * 4


def _desc(t: torch.Tensor | None) -> _Tensor:
    if t is None:
        return _Tensor()
    n = t.dim()
    if n > 4:
        raise ValueError("tensors passed to the library have at most 4 dimensions")
    pad = (0,) * (4 - n)
    return _Tensor(t.data_ptr() or None, _DTYPES.get(t.dtype, 0), n, _I64x4(*t.shape, *pad),
                   _I64x4(*t.stride(), *pad))


def _stream_handle(stream, device) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream or None
    return int(stream) or None


def workspace_size(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, num_splits: int = 0) -> int:
    """Bytes of workspace a call with these arguments needs (raises on invalid arguments)."""
    n = _load().apd_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, num_splits)
    if n == 0:
        raise ValueError("invalid arguments for apd_workspace_size "
                         f"(batch={batch}, Hq={num_q_heads}, Hkv={num_kv_heads}, D={head_dim}, splits={num_splits})")
    return int(n)


def alloc_workspace(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, num_splits: int = 0,
                    device="cuda") -> torch.Tensor:
    """A zeroed uint8 device buffer of workspace_size(...) bytes (torch allocations are 256-byte aligned)."""
    n = workspace_size(batch, num_q_heads, num_kv_heads, head_dim, num_splits)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def workspace_init(workspace: torch.Tensor, stream=None) -> None:
    rc = _load().apd_workspace_init(workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream_handle(stream, workspace.device))
    if rc:
        raise APDError(rc, "apd_workspace_init")


def attn_paged_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                      seq_lens: torch.Tensor, out: torch.Tensor, scale: float, num_splits: int = 0,
                      workspace: torch.Tensor | None = None, stream=None, split_done_event=None,
                      disable_pdl: bool = False, host_seq_lens=None) -> torch.Tensor:
    """out[b, h, :] = softmax(scale * q[b, h] . K_b^T) V_b over the paged cache; returns ``out``.

    q bf16 [B, Hq, D]; k_cache / v_cache bf16 [num_pages, page_size, Hkv, D] (any strides
    with D contiguous); page_table int32 [B, max_pages]; seq_lens int32 [B]; out bf16 [B, Hq, D].
    ``workspace``: a device buffer of at least workspace_size(...) bytes; preallocate it once
    (allocating here, when it is None, makes the call not capturable in a CUDA graph).
    ``split_done_event``: optional torch.cuda.Event recorded right after the split kernel.
    ``host_seq_lens``: optional host copy of the lengths (a planning hint with num_splits = 0;
    see apd_launch_options.host_seq_lens: it changes the launch, never the result).
    """
    L = _load()
    hl = _host_lens(host_seq_lens, q.shape[0])
    if workspace is None:
        workspace = alloc_workspace(q.shape[0], q.shape[1], k_cache.shape[2], q.shape[2], num_splits,
                                    device=q.device)
    descs = [_desc(t) for t in (q, k_cache, v_cache, page_table, seq_lens, out)]
    ptrs = [ctypes.byref(d) for d in descs]
    st = _stream_handle(stream, q.device)
    ws_ptr = workspace.data_ptr()
    ws_bytes = workspace.numel() * workspace.element_size()
    if split_done_event is None and not disable_pdl and hl is None:
        rc = L.apd_attn_paged_decode(*ptrs, ctypes.c_float(scale), int(num_splits), ws_ptr, ws_bytes, st)
    else:
        opts = _Options()
        opts.host_seq_lens = hl.data_ptr() if hl is not None else None
        if split_done_event is not None:
            if not split_done_event.cuda_event:  # torch creates its events lazily, at the first record
                split_done_event.record(torch.cuda.current_stream(q.device) if stream is None else stream)
            opts.split_done_event = split_done_event.cuda_event
        opts.disable_pdl = 1 if disable_pdl else 0
        rc = L.apd_attn_paged_decode_ex(*ptrs, ctypes.c_float(scale), int(num_splits), ws_ptr, ws_bytes, st,
                                        ctypes.byref(opts))
    if rc:
        raise APDError(rc, "apd_attn_paged_decode")
    return out


def attn_paged_decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                              page_table: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor, scale: float,
                              num_splits: int = 0, stream=None) -> torch.Tensor:
    """attn_paged_decode for callers that cannot allocate device memory: no workspace
    argument; the library's built-in static device scratch (NOALLOC_SCRATCH_BYTES per
    device, shared by every call, so calls must be ordered on the GPU) is used instead."""
    descs = [_desc(t) for t in (q, k_cache, v_cache, page_table, seq_lens, out)]
    rc = _load().apd_attn_paged_decode_noalloc(*[ctypes.byref(d) for d in descs], ctypes.c_float(scale),
                                               int(num_splits), _stream_handle(stream, q.device))
    if rc:
        raise APDError(rc, "apd_attn_paged_decode_noalloc")
    return out


def attn_contig_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seq_lens: torch.Tensor,
                       out: torch.Tensor, scale: float, num_splits: int = 0, workspace: torch.Tensor | None = None,
                       stream=None, host_seq_lens=None) -> torch.Tensor:
    """Decode attention over a contiguous KV cache: k / v bf16 [B, Lmax, Hkv, D] ("blhd"
    order; "bhld" storage is passed as the permuted view), token t of sequence b at
    k[b, t].  Same arguments and results as attn_paged_decode otherwise."""
    L = _load()
    if workspace is None:
        workspace = alloc_workspace(q.shape[0], q.shape[1], k.shape[2], q.shape[2], num_splits, device=q.device)
    descs = [_desc(t) for t in (q, k, v, seq_lens, out)]
    hl = _host_lens(host_seq_lens, q.shape[0])
    opts = _Options()
    opts.host_seq_lens = hl.data_ptr() if hl is not None else None
    rc = L.apd_attn_contig_decode_ex(*[ctypes.byref(d) for d in descs], ctypes.c_float(scale), int(num_splits),
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream_handle(stream, q.device), ctypes.byref(opts))
    if rc:
        raise APDError(rc, "apd_attn_contig_decode")
    return out


PREFILL_KERNELS = {"auto": 0, "mma_sync": 1, "tcgen05": 2}


def selftest_bounded_wait(short_timeout_ns: int = 1_000_000, device="cuda") -> list[int]:
    """Runs the library's bounded-wait self-test on the GPU and returns [first wait gave up,
    second wait gave up (through the abort flag), second wait's duration in us, flag word]."""
    out = torch.zeros(4, dtype=torch.int32, device=device)
    L = _load()
    rc = L.apd_selftest_bounded_wait(out.data_ptr(), int(short_timeout_ns), _stream_handle(None, out.device))
    if rc:
        raise APDError(rc, "apd_selftest_bounded_wait")
    torch.cuda.synchronize(out.device)
    return [int(v) & 0xFFFFFFFF for v in out.cpu().tolist()]


def selftest_shared_ring_release(q, k_cache, v_cache, page_table, seq_lens, out, scale: float,
                                 workspace: torch.Tensor, short_timeout_ns: int = 1_000_000, stream=None) -> None:
    """Enqueues the shared K/V ring's release self-test (apd_selftest_shared_ring_release) on
    a problem with more than 16 q heads per kv head: the followers never release a stage
    and every wait gives up after short_timeout_ns.  Read the outcome with
    read_device_flags(workspace)."""
    descs = [_desc(t) for t in (q, k_cache, v_cache, page_table, seq_lens, out)]
    rc = _load().apd_selftest_shared_ring_release(*[ctypes.byref(d) for d in descs], ctypes.c_float(scale),
                                                  workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                                  int(short_timeout_ns), _stream_handle(stream, q.device))
    if rc:
        raise APDError(rc, "apd_selftest_shared_ring_release")


def selftest_mq_tc_stall(q, k_cache, v_cache, page_table, seq_lens, out, scale: float, num_splits: int,
                         workspace: torch.Tensor, short_timeout_ns: int = 1_000_000, stream=None) -> None:
    """Enqueues the tensor-core multi-query kernel's stall self-test (apd_selftest_mq_tc_stall)
    on a problem that takes that kernel: the softmax warps never hand over the weights of their
    second tile and every wait gives up after short_timeout_ns.  Read the outcome with
    read_device_flags(workspace)."""
    descs = [_desc(t) for t in (q, k_cache, v_cache, page_table, seq_lens, out)]
    rc = _load().apd_selftest_mq_tc_stall(*[ctypes.byref(d) for d in descs], ctypes.c_float(scale), int(num_splits),
                                          workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                          int(short_timeout_ns), _stream_handle(stream, q.device))
    if rc:
        raise APDError(rc, "apd_selftest_mq_tc_stall")


def prefill_auto_kernel(head_dim: int) -> str:
    """The kernel attn_paged_prefill(kernel="auto") runs for a head dim."""
    return "tcgen05" if PREFILL_AUTO_TC else "mma_sync"


PREFILL_AUTO_TC = True  # mirrors the library's default choice


def attn_paged_prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                       seq_lens: torch.Tensor, scale: float, causal_offset: int = -1,
                       mask: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None,
                       kernel: str = "auto") -> torch.Tensor:
    """Multi-query attention of q [B, Lq, Hq, D] over the paged cache; returns out [B, Lq, Hq, D].

    causal_offset -1: no causal mask; c >= 0: query i sits at position c + i.  mask: None,
    uint8/bool [B, kv_len] or [B, Lq, kv_len] (nonzero = visible).  kernel: "auto",
    "mma_sync" or "tcgen05" (both: every head dim)."""
    if kernel not in PREFILL_KERNELS:
        raise ValueError(f"kernel must be one of {sorted(PREFILL_KERNELS)}")
    if out is None:
        out = torch.empty_like(q)
    if mask is not None and mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    L = _load()
    descs = [_desc(t) for t in (q, k_cache, v_cache, page_table, seq_lens)]
    md = _desc(mask) if mask is not None else None
    od = _desc(out)
    rc = L.apd_attn_paged_prefill_ex(*[ctypes.byref(d) for d in descs], ctypes.byref(md) if md is not None else None,
                                     ctypes.byref(od), ctypes.c_float(scale), int(causal_offset),
                                     _stream_handle(stream, q.device), PREFILL_KERNELS[kernel])
    if rc:
        raise APDError(rc, "apd_attn_paged_prefill")
    return out


def gemv_workspace_size(m: int, n: int, k: int) -> int:
    nb = _load().apd_gemv_workspace_size(m, n, k)
    if nb == 0:
        raise ValueError(f"invalid GEMV shape M={m}, N={n}, K={k}")
    return int(nb)


def gemv_query_plan(m: int, n: int, k: int, sm_count: int = 0) -> dict:
    """How apd_gemv_bf16 launches this shape (sm_count > 0: for a device with that many
    SMs, on the host; 0: the current device)."""
    p = _GemvPlan()
    rc = _load().apd_gemv_query_plan(m, n, k, int(sm_count), ctypes.byref(p))
    if rc:
        raise APDError(rc, "apd_gemv_query_plan")
    return {name: int(getattr(p, name)) for name, _ in _GemvPlan._fields_}


def gemv(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
         stream=None) -> torch.Tensor:
    """Decode projection y = x W^T: x bf16 [M, K] (M <= 8), w bf16 [N, K] -> y bf16 [M, N]."""
    if y is None:
        y = torch.empty(x.shape[0], w.shape[0], dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.zeros(gemv_workspace_size(x.shape[0], w.shape[0], x.shape[1]), dtype=torch.uint8,
                                device=x.device)
    d = [_desc(t) for t in (x, w, y)]
    rc = _load().apd_gemv_bf16(*[ctypes.byref(t) for t in d], workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream_handle(stream, x.device))
    if rc:
        raise APDError(rc, "apd_gemv_bf16")
    return y


class DecodeCall:
    """apd_attn_paged_decode with its arguments marshalled once, for repeated calls on
    the same buffers (a decode loop, a benchmark, a CUDA-graph capture).  Calling the
    object enqueues one decode call; the tensors' contents may change between calls,
    their storage, shapes and strides may not.  page_table=None selects the
    contiguous-KV call (apd_attn_contig_decode).  ``host_seq_lens``: the planning hint of
    attn_paged_decode, copied here and passed on every call."""

    def __init__(self, q, k_cache, v_cache, page_table, seq_lens, out, scale: float, num_splits: int = 0,
                 workspace: torch.Tensor | None = None, host_seq_lens=None):
        if workspace is None:
            workspace = alloc_workspace(q.shape[0], q.shape[1], k_cache.shape[2], q.shape[2], num_splits,
                                        device=q.device)
        self.tensors = (q, k_cache, v_cache, page_table, seq_lens, out, workspace)
        self.device = q.device
        self.contig = page_table is None
        args = (q, k_cache, v_cache, seq_lens, out) if self.contig else (q, k_cache, v_cache, page_table, seq_lens, out)
        self._descs = [_desc(t) for t in args]
        self._head = tuple(ctypes.byref(d) for d in self._descs) + (
            ctypes.c_float(scale), int(num_splits), workspace.data_ptr(), workspace.numel() * workspace.element_size())
        self._opts = _Options()
        self._host_lens = _host_lens(host_seq_lens, q.shape[0])
        self._opts.host_seq_lens = self._host_lens.data_ptr() if self._host_lens is not None else None
        self._opts_ref = ctypes.byref(self._opts)
        self._lib = _load()

    @property
    def out(self) -> torch.Tensor:
        return self.tensors[5]

    @property
    def workspace(self) -> torch.Tensor:
        return self.tensors[6]

    def __call__(self, stream=None, split_done_event=None) -> None:
        st = _stream_handle(stream, self.device)
        if split_done_event is None and self._host_lens is None:
            fn = self._lib.apd_attn_contig_decode if self.contig else self._lib.apd_attn_paged_decode
            rc = fn(*self._head, st)
        else:
            if split_done_event is not None and not split_done_event.cuda_event:
                # torch creates its events lazily, at the first record
                split_done_event.record(torch.cuda.current_stream(self.device) if stream is None else stream)
            self._opts.split_done_event = split_done_event.cuda_event if split_done_event is not None else None
            fn = self._lib.apd_attn_contig_decode_ex if self.contig else self._lib.apd_attn_paged_decode_ex
            rc = fn(*self._head, st, self._opts_ref)
        if rc:
            raise APDError(rc, "apd_attn_paged_decode")


def read_device_flags(workspace: torch.Tensor, clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return the sticky APD_FLAG_* word of the workspace."""
    flags = ctypes.c_uint32(0)
    rc = _load().apd_read_device_flags(workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                       _stream_handle(stream, workspace.device), ctypes.byref(flags),
                                       1 if clear else 0)
    if rc:
        raise APDError(rc, "apd_read_device_flags")
    return int(flags.value)


@dataclass
class Plan:
    mode: int
    num_workers: int
    grid_ctas: int
    warps_per_cta: int
    stages: int
    rows_per_unit: int
    head_blocks: int
    combine_ctas: int
    smem_bytes: int
    partial_slots: int
    workspace_bytes: int
    shared_kv_ring: int  # 1: a kv head's head-block warps read one K/V ring (balanced, g > 16)
    cluster_size: int = 0  # mode 3: CTAs per cluster that merge a unit's splits in the kernel
    q_head_blocks: int = 1  # mode 3: CTAs per split of a (sequence, kv head), one per block of q heads
    q_heads_per_block: int = 0  # mode 3: q heads of each block but the last (a multiple of 16)


def query_plan(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, num_splits: int = 0,
               workspace_bytes: int | None = None, sm_count: int = 0, host_seq_lens=None,
               max_seq_len: int = 0) -> Plan:
    """How the library would launch this problem (sm_count > 0: for a device with that
    many SMs, computed on the host; 0: for the current CUDA device).  With
    ``host_seq_lens`` (and ``max_seq_len`` = max_pages_per_seq * page_size, the clamp):
    the plan of a call given that hint."""
    p = _Plan()
    wb = ctypes.c_size_t(-1).value if workspace_bytes is None else int(workspace_bytes)
    hl = _host_lens(host_seq_lens, batch)
    rc = _load().apd_query_plan_ex(batch, num_q_heads, num_kv_heads, head_dim, num_splits, wb, int(sm_count),
                                   hl.data_ptr() if hl is not None else None, int(max_seq_len), ctypes.byref(p))
    if rc:
        raise APDError(rc, "apd_query_plan")
    return Plan(**{name: int(getattr(p, name)) for name, _ in _Plan._fields_ if not name.startswith("reserved")})
