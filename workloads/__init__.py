"""Seeded synthetic inputs for paged decode attention.

This module only *generates inputs*: bf16 query / KV-cache values, page tables and
sequence lengths.  It holds none of the attention arithmetic, so both the CPU
oracle (``oracle/``) and the CUDA library (``decode_attention_paged_split_b200``)
can be fed from it without sharing any of the method's code.

Recipe (the same everywhere; the seed is recorded by every caller):

* bf16 values are iid N(0, 1): fp32 draws from ``torch.randn`` rounded to bf16
  (round-to-nearest-even).  The flat tensor is cut into fixed chunks of
  ``_CHUNK`` elements; chunk ``c`` of stream ``s`` draws from a ``torch.Generator``
  seeded with ``SeedSequence([seed, s, c])``.  Chunks are filled in parallel
  threads, and the values do not depend on the thread count.
* Structure (sequence lengths, page permutation) comes from
  ``numpy.random.default_rng(seed)``.
* Page assignment: ``perm = rng.permutation(pool)``; sequence b takes the next
  ``ceil(L_b / P)`` pages of ``perm`` in order.
* KV cache layout is "NHD" ``[num_pages, page_size, kv_heads, head_dim]``.  The
  "HND" option allocates ``[num_pages, kv_heads, page_size, head_dim]`` storage
  and returns the NHD-ordered *view* of it (same logical tensor, other strides).
* ``poison=True`` writes NaN into every KV slot that a correct kernel must not
  read: the tail slots of each sequence's last page, every pool page that no
  sequence uses, and an extra all-NaN page that the unused page-table entries
  point at.  A read of any of them turns the output into NaN instead of
  faulting.

The workloads follow the shapes of the pages' decode cases (AstrAI commit log of
``csrc/kernels/attn_paged_decode.cu``: GQA, head_dim 32/64/128/256, multi-batch,
split-KV) scaled to the named decode configurations below.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

_CHUNK = 1 << 22  # elements per independently seeded chunk

# stream ids of the value tensors
_S_Q, _S_K, _S_V, _S_KMASK = 1, 2, 3, 4


@dataclass
class Workload:
    """One decode-attention problem, all tensors on the host (torch CPU)."""

    name: str
    seed: int
    q: torch.Tensor           # bf16 [B, Hq, D]
    k_cache: torch.Tensor     # bf16 [NP, P, Hkv, D] (a view, maybe strided)
    v_cache: torch.Tensor     # bf16 [NP, P, Hkv, D]
    page_table: torch.Tensor  # int32 [B, MP]
    seq_lens: torch.Tensor    # int32 [B]
    scale: float
    num_splits: int = 0
    layout: str = "NHD"
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def num_q_heads(self) -> int:
        return self.q.shape[1]

    @property
    def head_dim(self) -> int:
        return self.q.shape[2]

    @property
    def num_kv_heads(self) -> int:
        return self.k_cache.shape[2]

    @property
    def page_size(self) -> int:
        return self.k_cache.shape[1]

    @property
    def num_pages(self) -> int:
        return self.k_cache.shape[0]

    def kv_tokens(self) -> int:
        return int(self.seq_lens.to(torch.int64).sum())

    def algorithmic_bytes(self) -> int:
        """KV bytes that must be read + q bytes + out bytes (bf16)."""
        d, hkv, hq, b = self.head_dim, self.num_kv_heads, self.num_q_heads, self.batch
        return self.kv_tokens() * hkv * d * 2 * 2 + 2 * b * hq * d * 2

    def algorithmic_flops(self) -> int:
        """QK^T plus PV multiply-adds, 2 flops each."""
        return 4 * self.head_dim * self.num_q_heads * self.kv_tokens()

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "batch": self.batch,
            "num_q_heads": self.num_q_heads,
            "num_kv_heads": self.num_kv_heads,
            "head_dim": self.head_dim,
            "page_size": self.page_size,
            "num_pages": self.num_pages,
            "max_pages_per_seq": self.page_table.shape[1],
            "kv_tokens": self.kv_tokens(),
            "num_splits": self.num_splits,
            "layout": self.layout,
            "seed": self.seed,
            **self.meta,
        }


def _chunk_seed(seed: int, stream: int, chunk: int) -> int:
    return int(np.random.SeedSequence([seed, stream, chunk]).generate_state(1, dtype=np.uint64)[0]) >> 1


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def seeded_randn_bf16(numel: int, seed: int, stream: int) -> torch.Tensor:
    """Flat bf16 tensor of iid N(0,1) values; deterministic in (seed, stream)."""
    out = torch.empty(numel, dtype=torch.bfloat16)
    nchunks = (numel + _CHUNK - 1) // _CHUNK

    def fill(c: int) -> None:
        lo = c * _CHUNK
        hi = min(numel, lo + _CHUNK)
        g = torch.Generator().manual_seed(_chunk_seed(seed, stream, c))
        out[lo:hi].copy_(torch.randn(hi - lo, generator=g, dtype=torch.float32))

    if nchunks <= 1:
        for c in range(nchunks):
            fill(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def seeded_bernoulli(numel: int, p: float, seed: int, stream: int) -> torch.Tensor:
    """Flat bool tensor, each entry independently True with probability p."""
    out = torch.empty(numel, dtype=torch.bool)
    nchunks = (numel + _CHUNK - 1) // _CHUNK

    def fill(c: int) -> None:
        lo = c * _CHUNK
        hi = min(numel, lo + _CHUNK)
        g = torch.Generator().manual_seed(_chunk_seed(seed, stream, c))
        out[lo:hi].copy_(torch.rand(hi - lo, generator=g, dtype=torch.float32) < p)

    if nchunks <= 1:
        for c in range(nchunks):
            fill(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def make(
    *,
    name: str,
    seed: int,
    batch: int,
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    page_size: int,
    seq_lens,
    pool_pages: int | None = None,
    max_pages_per_seq: int | None = None,
    scale: float | None = None,
    num_splits: int = 0,
    k_outlier_frac: float = 0.0,
    k_outlier_mult: float = 8.0,
    layout: str = "NHD",
    poison: bool = False,
    meta: dict | None = None,
    value_seed: int | None = None,
) -> Workload:
    """Build one seeded problem.  ``seq_lens`` is a list/array of B ints.  ``seed`` drives
    the structure (page permutation); ``value_seed`` (default: ``seed``) drives the bf16
    values, so two problems can share their structure and differ in their data."""
    lens = np.asarray(seq_lens, dtype=np.int64).reshape(-1)
    assert lens.shape[0] == batch and (lens >= 0).all()
    P = page_size
    npages_seq = (lens + P - 1) // P
    used = int(npages_seq.sum())
    if pool_pages is None:
        pool_pages = used
    assert pool_pages >= used, "page pool too small for the sequences"
    mp = max_pages_per_seq if max_pages_per_seq is not None else max(1, int(npages_seq.max(initial=0)))
    assert mp >= int(npages_seq.max(initial=0))
    rng = np.random.default_rng(seed)
    perm = rng.permutation(pool_pages).astype(np.int64)

    total_pages = pool_pages + (1 if poison else 0)  # last page = all-NaN pad page
    pad_page = pool_pages if poison else 0
    pt = np.full((batch, mp), pad_page, dtype=np.int32)
    cursor = 0
    for b in range(batch):
        n = int(npages_seq[b])
        pt[b, :n] = perm[cursor:cursor + n]
        cursor += n

    vseed = seed if value_seed is None else value_seed
    q = seeded_randn_bf16(batch * num_q_heads * head_dim, vseed, _S_Q).view(batch, num_q_heads, head_dim)
    kv_numel = total_pages * P * num_kv_heads * head_dim
    if layout == "NHD":
        shape_store = (total_pages, P, num_kv_heads, head_dim)
        to_nhd = (0, 1, 2, 3)
    elif layout == "HND":
        shape_store = (total_pages, num_kv_heads, P, head_dim)
        to_nhd = (0, 2, 1, 3)
    else:
        raise ValueError(f"unknown layout {layout!r}")
    k_store = seeded_randn_bf16(kv_numel, vseed, _S_K).view(*shape_store)
    v_store = seeded_randn_bf16(kv_numel, vseed, _S_V).view(*shape_store)
    if k_outlier_frac > 0.0:
        mask = seeded_bernoulli(kv_numel, k_outlier_frac, vseed, _S_KMASK).view(*shape_store)
        k_store[mask] = k_store[mask] * k_outlier_mult  # x8 is exact in bf16
    k_cache = k_store.permute(*to_nhd)
    v_cache = v_store.permute(*to_nhd)

    if poison:
        nan = float("nan")
        k_cache[pool_pages] = nan
        v_cache[pool_pages] = nan
        in_use = np.zeros(pool_pages, dtype=bool)
        for b in range(batch):
            n = int(npages_seq[b])
            in_use[pt[b, :n]] = True
            tail = int(lens[b]) - (n - 1) * P if n > 0 else P
            if n > 0 and tail < P:
                last = int(pt[b, n - 1])
                k_cache[last, tail:] = nan
                v_cache[last, tail:] = nan
        unused = np.nonzero(~in_use)[0]
        if unused.size:
            idx = torch.from_numpy(unused)
            k_cache[idx] = nan
            v_cache[idx] = nan

    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return Workload(
        name=name,
        seed=seed,
        q=q,
        k_cache=k_cache,
        v_cache=v_cache,
        page_table=torch.from_numpy(pt),
        seq_lens=torch.from_numpy(lens.astype(np.int32)),
        scale=float(scale),
        num_splits=num_splits,
        layout=layout,
        meta=dict(meta or {}),
    )


def make_contig(
    *,
    name: str,
    seed: int,
    batch: int,
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    seq_lens,
    lmax: int | None = None,
    layout: str = "blhd",
    scale: float | None = None,
    value_seed: int | None = None,
    poison: bool = True,
    k_outlier_frac: float = 0.0,
) -> Workload:
    """A contiguous KV cache: k / v bf16 [B, Lmax, Hkv, D] ("blhd"), or "bhld" storage
    [B, Hkv, Lmax, D] returned as the [B, Lmax, Hkv, D]-ordered view.  Slots at or past a
    sequence's length hold NaN when ``poison`` (they must never be read).  The returned
    Workload describes the same cache as a paged one with one Lmax-token page per
    sequence (page_table[b] = [b]), which is how the oracle reads it."""
    lens = np.asarray(seq_lens, dtype=np.int64).reshape(-1)
    assert lens.shape[0] == batch and (lens >= 0).all()
    lmax = int(lmax if lmax is not None else max(1, int(lens.max(initial=0))))
    assert lmax >= int(lens.max(initial=0))
    vseed = seed if value_seed is None else value_seed
    q = seeded_randn_bf16(batch * num_q_heads * head_dim, vseed, _S_Q).view(batch, num_q_heads, head_dim)
    numel = batch * lmax * num_kv_heads * head_dim
    if layout == "blhd":
        shape_store, to_blhd = (batch, lmax, num_kv_heads, head_dim), (0, 1, 2, 3)
    elif layout == "bhld":
        shape_store, to_blhd = (batch, num_kv_heads, lmax, head_dim), (0, 2, 1, 3)
    else:
        raise ValueError(f"unknown layout {layout!r}")
    k = seeded_randn_bf16(numel, vseed, _S_K).view(*shape_store).permute(*to_blhd)
    v = seeded_randn_bf16(numel, vseed, _S_V).view(*shape_store).permute(*to_blhd)
    if k_outlier_frac > 0.0:
        mask = seeded_bernoulli(numel, k_outlier_frac, vseed, _S_KMASK).view(*shape_store).permute(*to_blhd)
        k[mask] = k[mask] * 8.0
    if poison:
        for b in range(batch):
            k[b, int(lens[b]):] = float("nan")
            v[b, int(lens[b]):] = float("nan")
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return Workload(name=name, seed=seed, q=q, k_cache=k, v_cache=v,
                    page_table=torch.arange(batch, dtype=torch.int32).view(batch, 1),
                    seq_lens=torch.from_numpy(lens.astype(np.int32)), scale=float(scale), layout=layout,
                    meta={"kv_policy": "contig", "lmax": lmax})


def paged_from_contig(w: Workload, page_size: int = 32, seed: int = 0, poison: bool = True) -> Workload:
    """The same tokens as a contiguous workload, placed page by page into a shuffled pool
    of ``page_size``-token pages (the pages' paged-versus-contiguous agreement case)."""
    B, Hkv, D = w.batch, w.num_kv_heads, w.head_dim
    lens = w.seq_lens.to(torch.int64).tolist()
    P = page_size
    npages = [(L + P - 1) // P for L in lens]
    pool = sum(npages)
    mp = max(1, max(npages, default=1))
    perm = np.random.default_rng([seed, 5]).permutation(max(pool, 1))
    fill = float("nan") if poison else 0.0
    k = torch.full((max(pool, 1), P, Hkv, D), fill, dtype=torch.bfloat16)
    v = torch.full((max(pool, 1), P, Hkv, D), fill, dtype=torch.bfloat16)
    pt = torch.zeros(B, mp, dtype=torch.int32)
    cursor = 0
    for b in range(B):
        for j in range(npages[b]):
            page = int(perm[cursor])
            cursor += 1
            pt[b, j] = page
            t0, t1 = j * P, min((j + 1) * P, lens[b])
            k[page, : t1 - t0] = w.k_cache[b, t0:t1]
            v[page, : t1 - t0] = w.v_cache[b, t0:t1]
    return Workload(name=w.name + "_paged", seed=w.seed, q=w.q, k_cache=k, v_cache=v, page_table=pt,
                    seq_lens=w.seq_lens, scale=w.scale, meta={"kv_policy": "paged"})


# ----------------------------------------------------------------------------
# The named decode workloads
# ----------------------------------------------------------------------------

def tiny(seed: int = 1234, **kw) -> Workload:
    """B=1, 4 q heads over 1 kv head, D=64, P=32, L=256 (8 pages) from a pool of 16."""
    args = dict(name="tiny_b1_h4x1_d64_l256", seed=seed, batch=1, num_q_heads=4, num_kv_heads=1,
                head_dim=64, page_size=32, seq_lens=[256], pool_pages=16, scale=1.0 / 8.0, num_splits=1)
    args.update(kw)
    return make(**args)


SWEEP_HEAD_DIMS = (32, 64, 128, 256)
SWEEP_HEADS = ((8, 8), (32, 8))
SWEEP_SPLITS = (1, 4)


def sweep_lengths(seed: int, batch: int = 4) -> np.ndarray:
    """Per-sequence lengths, integers uniform in [1, 1024] inclusive."""
    return np.random.default_rng([seed, 77]).integers(1, 1025, size=batch)


def sweep_case(head_dim: int, num_q_heads: int, num_kv_heads: int, num_splits: int,
               seed: int = 2024, **kw) -> Workload:
    """B=4, L_b ~ U{1..1024}, a seeded shuffle of a 512-page pool."""
    args = dict(name=f"sweep_d{head_dim}_h{num_q_heads}x{num_kv_heads}_s{num_splits}", seed=seed,
                batch=4, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                page_size=32, seq_lens=sweep_lengths(seed), pool_pages=512, max_pages_per_seq=32,
                num_splits=num_splits)
    args.update(kw)
    return make(**args)


def sweep_cases():
    for d in SWEEP_HEAD_DIMS:
        for hq, hkv in SWEEP_HEADS:
            for s in SWEEP_SPLITS:
                yield d, hq, hkv, s


def llama8b(seed: int = 8, **kw) -> Workload:
    """B=16, 32 q heads / 8 kv heads, D=128, L=4096 each, 2048-page shuffled pool,
    1% of K entries scaled x8."""
    args = dict(name="llama8b_b16_h32x8_d128_l4096", seed=seed, batch=16, num_q_heads=32,
                num_kv_heads=8, head_dim=128, page_size=32, seq_lens=[4096] * 16, pool_pages=2048,
                num_splits=0, k_outlier_frac=0.01, k_outlier_mult=8.0)
    args.update(kw)
    return make(**args)


def long_context(seed: int = 131072, **kw) -> Workload:
    """B=2, 32 q heads / 8 kv heads, D=128, L=131072 (4096 pages each), shuffled."""
    args = dict(name="long_b2_h32x8_d128_l131072", seed=seed, batch=2, num_q_heads=32,
                num_kv_heads=8, head_dim=128, page_size=32, seq_lens=[131072] * 2,
                pool_pages=8192, num_splits=0)
    args.update(kw)
    return make(**args)


def ragged_lengths(seed: int, batch: int = 128, lo: int = 16, hi: int = 32768) -> np.ndarray:
    """floor(exp(U(ln lo, ln(hi+1)))) clamped to [lo, hi] (log-uniform integers)."""
    u = np.random.default_rng([seed, 99]).uniform(math.log(lo), math.log(hi + 1), size=batch)
    return np.clip(np.floor(np.exp(u)).astype(np.int64), lo, hi)


def ragged(seed: int = 4262, **kw) -> Workload:
    """B=128, 64 q heads / 8 kv heads, D=128, L_b log-uniform in [16, 32768],
    one shared shuffled pool sized to the total."""
    lens = ragged_lengths(seed)
    args = dict(name="ragged_b128_h64x8_d128_loguniform16_32768", seed=seed, batch=128,
                num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=32, seq_lens=lens,
                max_pages_per_seq=1024, num_splits=0)
    args.update(kw)
    return make(**args)


def llama8b_contig(seed: int = 8, **kw) -> Workload:
    """The llama8b-shaped decode over a contiguous [16, 4096, 8, 128] KV cache."""
    args = dict(name="llama8b_contig_b16_h32x8_d128_l4096", seed=seed, batch=16, num_q_heads=32, num_kv_heads=8,
                head_dim=128, seq_lens=[4096] * 16, lmax=4096, k_outlier_frac=0.01, poison=False)
    args.update(kw)
    return make_contig(**args)


def long_contig(seed: int = 131072, **kw) -> Workload:
    """The long-context decode over a contiguous [2, 131072, 8, 128] KV cache."""
    args = dict(name="long_contig_b2_h32x8_d128_l131072", seed=seed, batch=2, num_q_heads=32, num_kv_heads=8,
                head_dim=128, seq_lens=[131072] * 2, lmax=131072, poison=False)
    args.update(kw)
    return make_contig(**args)


def gqa32(seed: int = 32, **kw) -> Workload:
    """B=16, 64 q heads / 2 kv heads (32 q heads per kv head: two 16-row head blocks),
    D=128, L=16384 each (268 MB of K/V, the llama8b byte count), shuffled pool."""
    args = dict(name="gqa32_b16_h64x2_d128_l16384", seed=seed, batch=16, num_q_heads=64,
                num_kv_heads=2, head_dim=128, page_size=32, seq_lens=[16384] * 16, pool_pages=8192,
                num_splits=0)
    args.update(kw)
    return make(**args)


def gqa80(seed: int = 80, **kw) -> Workload:
    """B=16, 80 q heads / 1 kv head (two blocks of q heads for the tensor-core decode), D=128,
    L=32768 each (268 MB of K/V, the llama8b byte count), shuffled pool."""
    args = dict(name="gqa80_b16_h80x1_d128_l32768", seed=seed, batch=16, num_q_heads=80,
                num_kv_heads=1, head_dim=128, page_size=32, seq_lens=[32768] * 16, pool_pages=16384,
                num_splits=0)
    args.update(kw)
    return make(**args)


def head_dim_scale(head_dim: int, seed: int = 77, **kw) -> Workload:
    """The llama8b shape (B=16, 32 q heads / 8 kv heads) at another head dim, with the
    sequence length that keeps 268 MB of K/V: L = 4096 * 128 / D, shuffled pool."""
    L = 4096 * 128 // head_dim
    args = dict(name=f"hd{head_dim}_b16_h32x8_d{head_dim}_l{L}", seed=seed, batch=16, num_q_heads=32,
                num_kv_heads=8, head_dim=head_dim, page_size=32, seq_lens=[L] * 16, pool_pages=16 * L // 32,
                num_splits=0)
    args.update(kw)
    return make(**args)


NAMED = {
    "tiny": tiny,
    "llama8b": llama8b,
    "long": long_context,
    "ragged": ragged,
    "gqa32": gqa32,
    "gqa80": gqa80,
    "llama8b_contig": llama8b_contig,
    "long_contig": long_contig,
    "hd32": lambda seed=77, **kw: head_dim_scale(32, seed, **kw),
    "hd64": lambda seed=77, **kw: head_dim_scale(64, seed, **kw),
    "hd256": lambda seed=77, **kw: head_dim_scale(256, seed, **kw),
}


# ----------------------------------------------------------------------------
# Decode projection (GEMV) inputs: x [M, K] and W [N, K] bf16, iid N(0, 1)
# ----------------------------------------------------------------------------
_S_GX, _S_GW = 11, 12

# (N, K) of the projections of the AstrAI 1B decode benchmark (hidden 1536,
# intermediate 6912, vocabulary 100000, kv width 256), named after their layers.
GEMV_SHAPES = {
    "q": (1536, 1536),
    "kv": (256, 1536),
    "gate_up": (6912, 1536),
    "down": (1536, 6912),
    "lm_head": (100000, 1536),
}


@dataclass
class GemvCase:
    name: str
    seed: int
    x: torch.Tensor  # bf16 [M, K]
    w: torch.Tensor  # bf16 [N, K]

    def algorithmic_bytes(self) -> int:
        """Weight bytes + x bytes + y bytes (bf16)."""
        M, K = self.x.shape
        N = self.w.shape[0]
        return 2 * (N * K + M * K + M * N)

    def algorithmic_flops(self) -> int:
        M, K = self.x.shape
        return 2 * M * K * self.w.shape[0]


def gemv_case(M: int, N: int, K: int, seed: int = 7, name: str | None = None, value_seed: int | None = None) -> GemvCase:
    vs = seed if value_seed is None else value_seed
    x = seeded_randn_bf16(M * K, vs, _S_GX).view(M, K)
    w = seeded_randn_bf16(N * K, vs, _S_GW).view(N, K)
    return GemvCase(name=name or f"gemv_m{M}_n{N}_k{K}", seed=seed, x=x, w=w)


def gemv_named(layer: str, M: int, seed: int = 7, **kw) -> GemvCase:
    N, K = GEMV_SHAPES[layer]
    return gemv_case(M, N, K, seed=seed, name=f"gemv_{layer}_m{M}_n{N}_k{K}", **kw)


# ----------------------------------------------------------------------------
# Multi-query (chunked prefill) inputs over the same paged cache
# ----------------------------------------------------------------------------
_S_PQ, _S_MASK = 13, 14


@dataclass
class PrefillWorkload:
    """Lq query tokens per sequence against a paged cache (all host tensors)."""

    name: str
    seed: int
    q: torch.Tensor            # bf16 [B, Lq, Hq, D]
    k_cache: torch.Tensor      # bf16 [NP, P, Hkv, D]
    v_cache: torch.Tensor
    page_table: torch.Tensor   # int32 [B, MP]
    seq_lens: torch.Tensor     # int32 [B]
    scale: float
    causal_offset: int = -1    # -1: no causal mask; c >= 0: query i sits at position c + i
    mask: torch.Tensor | None = None  # uint8 [B, kv_len] or [B, Lq, kv_len]; nonzero = visible

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def q_len(self) -> int:
        return self.q.shape[1]

    def algorithmic_bytes(self) -> int:
        """KV bytes of the visible range of every sequence + q + out (bf16)."""
        B, Lq, Hq, D = self.q.shape
        Hkv = self.k_cache.shape[2]
        kv = 0
        for b in range(B):
            L = int(self.seq_lens[b])
            if self.causal_offset >= 0:
                L = min(L, self.causal_offset + Lq)
            kv += L
        return kv * Hkv * D * 4 + 2 * B * Lq * Hq * D * 2

    def algorithmic_flops(self) -> int:
        """QK^T + PV over the (query, key) pairs each query sees without a mask."""
        B, Lq, Hq, D = self.q.shape
        pairs = 0
        for b in range(B):
            L = int(self.seq_lens[b])
            for i in range(Lq):
                pairs += L if self.causal_offset < 0 else max(0, min(L, self.causal_offset + i + 1))
        return 4 * D * Hq * pairs


def make_prefill(*, name: str, seed: int, batch: int, q_len: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, seq_lens, page_size: int = 32, causal_offset: int = -1, mask: str | None = None,
                 mask_keep: float = 0.9, layout: str = "NHD", poison: bool = False, pool_pages: int | None = None,
                 max_pages_per_seq: int | None = None, scale: float | None = None) -> PrefillWorkload:
    """``mask``: None, "2d" ([B, kv_len]) or "3d" ([B, Lq, kv_len]), each entry visible
    with probability ``mask_keep`` (seeded), kv_len = max_pages_per_seq * page_size."""
    base = make(name=name, seed=seed, batch=batch, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                head_dim=head_dim, page_size=page_size, seq_lens=seq_lens, pool_pages=pool_pages,
                max_pages_per_seq=max_pages_per_seq, scale=scale, layout=layout, poison=poison)
    q = seeded_randn_bf16(batch * q_len * num_q_heads * head_dim, seed, _S_PQ).view(
        batch, q_len, num_q_heads, head_dim)
    m = None
    if mask is not None:
        kv_len = base.page_table.shape[1] * page_size
        shape = (batch, kv_len) if mask == "2d" else (batch, q_len, kv_len)
        n = int(np.prod(shape))
        keep = seeded_bernoulli(n, mask_keep, seed, _S_MASK).view(*shape)
        m = keep.to(torch.uint8)
    return PrefillWorkload(name=name, seed=seed, q=q, k_cache=base.k_cache, v_cache=base.v_cache,
                           page_table=base.page_table, seq_lens=base.seq_lens, scale=base.scale,
                           causal_offset=causal_offset, mask=m)


def prefill_llama8b_chunk(seed: int = 8, **kw) -> PrefillWorkload:
    """A 128-token prefill chunk at the end of 16 sequences of 4096 keys, 32/8 heads,
    D = 128, causal (queries at positions 3968..4095), over a shuffled 2048-page pool."""
    args = dict(name="prefill_llama8b_b16_q128_h32x8_d128_l4096", seed=seed, batch=16, q_len=128, num_q_heads=32,
                num_kv_heads=8, head_dim=128, seq_lens=[4096] * 16, page_size=32, causal_offset=4096 - 128,
                pool_pages=2048)
    args.update(kw)
    return make_prefill(**args)
