"""Host-only checks of the C-ABI library: it loads, exports every symbol its
header declares, rejects bad arguments with the documented status codes before
touching the GPU, and plans launches as documented.  No test here needs a GPU or
launches a kernel.
"""
import ctypes
import os
import re

import pytest
import torch
from hypothesis import given, settings, strategies as st

import decode_attention_paged_split_b200 as apd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_paged_decode.h")

OK, NULLP, DTYPE, SHAPE, GQA, HEADDIM, LAYOUT, PAGESIZE, NSPLIT, WS, TOOLARGE, CUDA, ARG = range(13)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(apd_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("apd_attn_paged_decode", "apd_workspace_size", "apd_status_string", "apd_attn_paged_decode_ex",
                 "apd_attn_contig_decode",
                 "apd_query_plan", "apd_workspace_init", "apd_read_device_flags", "apd_last_cuda_error"):
        assert must in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(apd.library_path())
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings():
    for code in range(14):
        s = apd.status_string(code)
        assert s and s != "unknown status"
    assert apd.status_string(999) == "unknown status"


# ---------------------------------------------------------------- fake descriptors
FAKE = 1 << 32  # never dereferenced: every case below fails validation first


def T(shape, dtype=apd.DTYPE_BF16, stride=None, data=FAKE):
    d = apd._Tensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    if stride is None:
        stride, acc = [], 1
        for s in reversed(shape):
            stride.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, stride)):
        d.shape[i] = s
        d.stride[i] = st
    return d


def problem(B=2, Hq=8, Hkv=2, D=64, P=32, NP=16, MP=4):
    return dict(
        q=T([B, Hq, D]), k=T([NP, P, Hkv, D]), v=T([NP, P, Hkv, D]),
        pt=T([B, MP], apd.DTYPE_INT32), sl=T([B], apd.DTYPE_INT32), out=T([B, Hq, D]),
    )


def call(p, splits=0, ws=FAKE, ws_bytes=1 << 30, scale=0.125):
    L = apd.lib()
    return L.apd_attn_paged_decode(ctypes.byref(p["q"]), ctypes.byref(p["k"]), ctypes.byref(p["v"]),
                                   ctypes.byref(p["pt"]), ctypes.byref(p["sl"]), ctypes.byref(p["out"]),
                                   ctypes.c_float(scale), splits, ws, ws_bytes, None)


@pytest.mark.parametrize("field", ["q", "k", "v", "pt", "sl", "out"])
def test_null_pointer(field):
    p = problem()
    p[field].data = None
    assert call(p) == NULLP


def test_null_descriptor():
    p = problem()
    L = apd.lib()
    rc = L.apd_attn_paged_decode(None, ctypes.byref(p["k"]), ctypes.byref(p["v"]), ctypes.byref(p["pt"]),
                                 ctypes.byref(p["sl"]), ctypes.byref(p["out"]), ctypes.c_float(1.0), 0, FAKE,
                                 1 << 30, None)
    assert rc == NULLP


@pytest.mark.parametrize("field,dtype", [("q", apd.DTYPE_FP32), ("k", apd.DTYPE_INT32), ("v", apd.DTYPE_FP32),
                                         ("out", apd.DTYPE_FP32), ("pt", apd.DTYPE_BF16), ("sl", apd.DTYPE_FP32)])
def test_dtype(field, dtype):
    p = problem()
    p[field].dtype = dtype
    assert call(p) == DTYPE


def test_shape_errors():
    p = problem()
    p["q"] = T([2, 8, 64, 1])
    assert call(p) == SHAPE
    p = problem()
    p["out"] = T([2, 8, 32])
    assert call(p) == SHAPE
    p = problem()
    p["v"] = T([16, 32, 2, 32])
    assert call(p) == SHAPE
    p = problem()
    p["pt"] = T([3, 4], apd.DTYPE_INT32)
    assert call(p) == SHAPE
    p = problem()
    p["sl"] = T([3], apd.DTYPE_INT32)
    assert call(p) == SHAPE


def test_gqa_divisibility():
    p = problem(Hq=6, Hkv=4)
    assert call(p) == GQA


@pytest.mark.parametrize("D", [16, 48, 96, 512])
def test_head_dim(D):
    assert call(problem(D=D)) == HEADDIM


@pytest.mark.parametrize("P", [16, 48, 8])
def test_page_size(P):
    assert call(problem(P=P)) == PAGESIZE


def test_layout_errors():
    p = problem()
    p["q"] = T([2, 8, 64], stride=[512, 1, 8])  # head dim not contiguous
    assert call(p) == LAYOUT
    p = problem()
    p["k"] = T([16, 32, 2, 64], stride=[32 * 2 * 68, 2 * 68, 68, 1])  # 68 elements: not 16-byte aligned
    assert call(p) == LAYOUT
    p = problem()
    p["out"].data = FAKE + 2  # misaligned base
    assert call(p) == LAYOUT
    p = problem()
    p["sl"] = T([2], apd.DTYPE_INT32, stride=[2])
    assert call(p) == LAYOUT


def test_hnd_strides_are_accepted_by_validation():
    """HND storage [NP, Hkv, P, D] passed as the NHD-ordered view passes the checks
    (the call then needs a device, which this host does not have)."""
    NP, P, Hkv, D = 16, 32, 2, 64
    p = problem()
    p["k"] = T([NP, P, Hkv, D], stride=[Hkv * P * D, D, P * D, 1])
    p["v"] = T([NP, P, Hkv, D], stride=[Hkv * P * D, D, P * D, 1])
    assert call(p, ws_bytes=1 << 30) in (OK, CUDA)


def test_num_splits_negative():
    assert call(problem(), splits=-1) == NSPLIT


def test_workspace_errors():
    assert call(problem(), ws=None) == WS
    assert call(problem(), ws=FAKE + 128) == WS
    assert call(problem(), splits=4, ws_bytes=1024) == WS


def test_batch_too_large():
    assert call(problem(B=5000)) == TOOLARGE


def test_empty_batch_is_a_no_op():
    assert call(problem(B=0)) == OK


def test_ex_reserved_must_be_zero():
    p = problem()
    opts = apd._Options()
    opts.reserved = 1
    L = apd.lib()
    rc = L.apd_attn_paged_decode_ex(ctypes.byref(p["q"]), ctypes.byref(p["k"]), ctypes.byref(p["v"]),
                                    ctypes.byref(p["pt"]), ctypes.byref(p["sl"]), ctypes.byref(p["out"]),
                                    ctypes.c_float(1.0), 0, FAKE, 1 << 30, None, ctypes.byref(opts))
    assert rc == ARG


# ---------------------------------------------------------------- planning
def test_workspace_size_invalid_is_zero():
    L = apd.lib()
    assert L.apd_workspace_size(2, 6, 4, 64, 0) == 0
    assert L.apd_workspace_size(2, 8, 2, 80, 0) == 0
    assert L.apd_workspace_size(2, 8, 2, 64, -1) == 0
    with pytest.raises(ValueError):
        apd.workspace_size(2, 6, 4, 64)


def test_plan_struct_layout():
    # the C struct apd_plan and its ctypes mirror: 8 int32, 3 int64, 4 int32
    assert ctypes.sizeof(apd._Plan) == 72 and apd._Plan.q_heads_per_block.offset == 68


@pytest.mark.parametrize("B,Hq,Hkv,D", [(16, 32, 8, 128), (2, 32, 8, 128), (128, 64, 8, 128), (4, 8, 8, 32),
                                        (4, 32, 8, 256), (3, 40, 2, 64), (16, 64, 2, 64), (8, 160, 2, 64)])
def test_plan_balanced_fills_the_device(B, Hq, Hkv, D):
    pl = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=148)
    g = Hq // Hkv
    ups = Hkv * -(-g // 16)  # warps per group: one per (kv head, 16-row head block)
    assert pl.mode == 0
    # as many whole groups as the warp budget holds (7/8 of the resident warps for
    # D = 128, all of them otherwise): at most one CTA per SM
    budget = 148 * pl.warps_per_cta * 7 // 8 if D == 128 else 148 * pl.warps_per_cta
    assert pl.num_workers == (budget // ups) * ups
    assert pl.grid_ctas == -(-pl.num_workers // pl.warps_per_cta) <= 148
    assert budget - pl.num_workers < ups
    assert pl.partial_slots == 2 * pl.num_workers
    assert pl.rows_per_unit == min(g, 16) and pl.head_blocks == -(-g // 16)
    # when a unit has at most one batch of 4 partials (about groups / B + 1): up to 4
    # combine CTAs per SM walking the units; else one per (unit, row)
    per_unit = pl.num_workers // ups // B + 1 <= 4
    units = B * Hkv * pl.head_blocks
    assert pl.combine_ctas == (min(units, 4 * 148) if per_unit else units * pl.rows_per_unit)
    assert pl.smem_bytes <= 232448
    assert pl.workspace_bytes % 256 == 0
    assert pl.workspace_bytes == apd.lib().apd_workspace_size(B, Hq, Hkv, D, 0)


# per head dim: async-copy stages and the most warps a CTA may have, with one ring per
# warp and with a K/V ring shared by the head blocks of a kv head (None: not shared)
_TRAITS = {32: (3, 12), 64: (2, 10), 128: (3, 6), 256: (2, 4)}
# the unit kernel (one CTA per unit, or per fixed split): 16 warps x 2 stages at D = 32
_UNIT_TRAITS = {**_TRAITS, 32: (2, 16)}
_SHARE_TRAITS = {32: None, 64: (4, 8), 128: (2, 8), 256: (2, 4)}


def _smem(B, D, rows, warps, stages, hb, shared):
    """Dynamic shared memory of the split kernel: mbarriers (full, plus empty when the K/V
    ring is shared), the CTA's abort word (8 bytes), lengths and prefix sums, 1 KB of
    alignment slack, then the rings: per warp [K | V | Q] stages, or, shared, one K/V ring
    per kv head and one Q ring per warp (K and V tiles are 32 tokens x D bf16, Q tiles 1 KB
    aligned)."""
    meta = 8 * warps * stages * (2 if shared else 1) + 8 + 4 * (2 * B + 1)
    kv = 2 * 32 * D * 2
    q = -(-rows * D * 2 // 1024) * 1024
    rings = (warps // hb * stages * kv + warps * stages * q) if shared else warps * stages * (kv + q)
    return -(-meta // 16) * 16 + 1024 + rings


@pytest.mark.parametrize("B,Hq,Hkv,D", [(4, 160, 2, 64), (4, 192, 2, 256), (4, 64, 1, 64), (4, 80, 1, 32),
                                        (4, 64, 2, 256), (4, 32, 8, 128), (4, 16, 1, 64)])
def test_plan_shared_kv_ring(B, Hq, Hkv, D):
    # balanced mode with g > 16: the head blocks of a kv head share one K/V ring, so the
    # warps per CTA are the most that fit which are a multiple of the head blocks
    g = Hq // Hkv
    hb, rows = -(-g // 16), min(g, 16)

    def fits(shared):
        stages, max_warps = _SHARE_TRAITS[D] if shared else _TRAITS[D]
        return stages, [w for w in range(max_warps, 0, -1)
                        if (not shared or w % hb == 0) and _smem(B, D, rows, w, stages, hb, shared) <= 232448]

    shared = hb > 1 and _SHARE_TRAITS[D] is not None and bool(fits(True)[1])
    stages, ws = fits(shared)
    pl = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=148)
    assert pl.shared_kv_ring == int(shared)
    assert pl.warps_per_cta == ws[0] and pl.stages == stages
    assert pl.smem_bytes == _smem(B, D, rows, ws[0], stages, hb, shared)
    # fixed splits and the one-CTA-per-unit plan run the unit kernel: one ring per warp
    stages, max_warps = _UNIT_TRAITS[D]
    uw = max(x for x in range(1, max_warps + 1) if _unit_smem(D, rows, x, stages) <= 232448)
    fixed = apd.query_plan(B, Hq, Hkv, D, 2, sm_count=148)
    assert fixed.shared_kv_ring == 0 and fixed.stages == stages and fixed.warps_per_cta == uw
    assert fixed.smem_bytes == _unit_smem(D, rows, uw, stages)
    local = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=148, host_seq_lens=[4096] * B, max_seq_len=4096)
    if local.mode == 2:
        assert local.shared_kv_ring == 0 and local.stages == stages
        assert local.smem_bytes == _unit_smem(D, rows, local.warps_per_cta, stages)


def _mc_smem(nh):
    """Shared memory of the tensor-core multi-query kernel: the header (2 KB at 32 heads,
    1.75 KB at 64), 1 KB of alignment slack, Q [nh][128], 3 K and 3 V stages of 128 tokens x
    128, and two P buffers [128][nh] (bf16) at 32 heads, one at 64."""
    header, p_buffers = (2048, 2) if nh == 32 else (1792, 1)
    return header + 1024 + nh * 128 * 2 + 6 * 128 * 128 * 2 + p_buffers * 128 * nh * 2


@pytest.mark.parametrize("g", [32, 20, 48, 64, 65, 80, 96, 128, 200])
@pytest.mark.parametrize("B,Hkv,sm", [(16, 2, 148), (1, 1, 148), (4, 8, 148), (200, 1, 148), (3, 2, 132), (16, 2, 8)])
def test_plan_tensor_core_multi_query(B, Hkv, sm, g):
    """More than 16 q heads per kv head at D = 128: the tensor-core multi-query kernel.
    The q heads of a kv head form nb = ceil(g / 64) blocks of ceil(g / nb) heads rounded
    up to 16 (the last block takes the rest), each padded to 32 or 64; one CTA per split of
    each (sequence, kv head, block), 7 or 11 warps (4 softmax warps per 32 heads, 2
    producers, 1 MMA issuer), K and V rings of 128-token stages, Q and two P buffers in
    shared memory.  Auto splits spread the (sequence, kv head, block) units over 7/8 of the
    SMs.  A unit's splits (up to 8) that the device can run as one cluster merge over DSMEM
    in the kernel; otherwise their partials take the fixed-split slots of the 16-row head
    blocks and the combine kernel merges them.  The slots are reserved either way."""
    Hq, D = g * Hkv, 128
    nb = -(-g // 64)
    per_block = -(-(-(-g // nb)) // 16) * 16
    assert per_block <= 64 and (nb - 1) * per_block < g
    nh = 32 if per_block <= 32 else 64
    units = B * Hkv * -(-g // 16)
    pl = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=sm)
    k = max(1, sm * 7 // 8 // (B * Hkv * nb))
    assert pl.mode == 3 and pl.shared_kv_ring == 0
    assert pl.q_head_blocks == nb and pl.q_heads_per_block == per_block
    assert pl.grid_ctas == B * Hkv * nb * k and pl.num_workers == pl.grid_ctas
    # a softmax group of 4 warps per 32 heads, 2 producer warps and the MMA issuer's warp
    assert pl.warps_per_cta == 4 * (nh // 32) + 3 and pl.stages == 3
    assert pl.smem_bytes == _mc_smem(nh) <= 232448
    assert pl.rows_per_unit == 16 and pl.head_blocks == -(-g // 16)
    assert pl.partial_slots == (units * k if k > 1 else 0)
    # up to 8 splits of a unit that fit the device as one cluster each merge in the kernel
    # (with an SM count given, every k SMs are taken to hold a cluster of k)
    cl = k if 2 <= k <= 8 and B * Hkv * nb <= sm // k else 0
    assert pl.cluster_size == cl
    assert pl.combine_ctas == (0 if k == 1 or cl else min(units, 4 * sm) if k <= 4 else units * 16)
    for S in (1, 3, 8, 12):
        f = apd.query_plan(B, Hq, Hkv, D, S, sm_count=sm)
        assert f.mode == 3 and f.grid_ctas == B * Hkv * nb * S and f.partial_slots == (units * S if S > 1 else 0)
        assert f.cluster_size == (S if 2 <= S <= 8 and B * Hkv * nb <= sm // S else 0)
    # a workspace that holds fewer partials caps the splits; one with none gives one split
    small = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=sm, workspace_bytes=4096)
    assert small.mode == 3 and small.grid_ctas == B * Hkv * nb and small.partial_slots == 0
    # other head dims and group sizes keep the mma.sync kernels
    for Hq2, D2 in ((g * Hkv, 64), (g * Hkv, 256), (16 * Hkv, 128)):
        assert apd.query_plan(B, Hq2, Hkv, D2, 0, sm_count=sm).mode != 3


def _unit_smem(D, rows, warps, stages):
    """Dynamic shared memory of the one-CTA-per-unit kernel: full mbarriers, the merge
    mbarrier, the abort word and tile counter (8 bytes), the claimed tile of each stage,
    1 KB of alignment slack, then one [K | V | Q] ring per warp."""
    meta = 8 * warps * stages + 8 + 8 + 4 * warps * stages
    q = -(-rows * D * 2 // 1024) * 1024
    return -(-meta // 16) * 16 + 1024 + warps * stages * (2 * 32 * D * 2 + q)


@pytest.mark.parametrize("B,Hq,Hkv,D,L", [(16, 32, 8, 128, 4096), (18, 16, 8, 64, 3000), (1, 4, 1, 64, 256),
                                          (16, 8, 8, 32, 1024), (32, 16, 4, 256, 1024)])
def test_plan_unit_kernel_smem(B, Hq, Hkv, D, L):
    """With host lengths that give one CTA per unit: the most warps (up to the head dim's
    maximum) whose rings fit, and the unit kernel's shared-memory layout."""
    pl = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=148, host_seq_lens=[L] * B, max_seq_len=L)
    assert pl.mode == 2
    stages, max_warps = _UNIT_TRAITS[D]
    rows = min(Hq // Hkv, 16)
    w = max(x for x in range(1, max_warps + 1) if _unit_smem(D, rows, x, stages) <= 232448)
    assert pl.warps_per_cta == w and pl.stages == stages
    assert pl.smem_bytes == _unit_smem(D, rows, w, stages)


@pytest.mark.parametrize("splits", [1, 2, 4, 148])
def test_plan_fixed(splits):
    B, Hq, Hkv, D = 16, 32, 8, 128
    pl = apd.query_plan(B, Hq, Hkv, D, splits, sm_count=148)
    units = B * Hkv
    assert pl.mode == 1
    # one unit-kernel CTA per split of each unit
    assert pl.grid_ctas == units * splits
    assert pl.num_workers == pl.grid_ctas * pl.warps_per_cta
    assert pl.partial_slots == (units * splits if splits > 1 else 0)
    assert pl.combine_ctas == ((min(units, 4 * 148) if splits <= 4 else units * pl.rows_per_unit) if splits > 1 else 0)
    assert pl.workspace_bytes == apd.workspace_size(B, Hq, Hkv, D, splits)


def test_plan_small_workspace_uses_fewer_workers():
    B, Hq, Hkv, D = 16, 32, 8, 128
    full = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=148)
    half = apd.query_plan(B, Hq, Hkv, D, 0, workspace_bytes=full.workspace_bytes // 2, sm_count=148)
    assert 0 < half.num_workers < full.num_workers
    assert half.workspace_bytes <= full.workspace_bytes // 2


def cta_local_expected(B, Hq, Hkv, D, lens, cap, sm=148):
    """The one-CTA-per-unit choice restated from its rule: every unit on its own SM, one
    head block per kv head, and the longest unit within 3% plus 1024 / D tiles of the share
    per CTA of a launch on max(units, 7/8 of the SMs) CTAs."""
    base = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=sm)
    units = B * Hkv * base.head_blocks
    tiles = [-(-min(max(L, 0), cap) // 32) for L in lens]
    total = sum(tiles) * Hkv * base.head_blocks
    share = -(-total // max(units, sm * 7 // 8))
    return (units <= sm and base.head_blocks == 1 and base.combine_ctas > 0
            and 32 * max(tiles) <= 33 * share + 32 * (1024 // D))


@pytest.mark.parametrize("B,Hq,Hkv,D,lens,cap,want", [
    (16, 32, 8, 128, [4096] * 16, 4096, 2),            # the LLaMA-8B-shaped batch: 128 units, one per CTA
    (16, 32, 8, 128, [4000] * 15 + [4096], 4096, 2),   # within the slack
    (16, 32, 8, 128, [2048] * 15 + [4096], 4096, 0),   # one long sequence: balanced
    (2, 32, 8, 128, [131072] * 2, 131072, 0),          # 16 units on 128 CTAs: balanced
    (128, 64, 8, 128, [1000] * 128, 1024, 0),          # 1024 units > SMs: balanced
    (18, 32, 8, 128, [4096] * 18, 4096, 2),            # 144 units: 128 tiles each, under the 144-tile share
    (20, 32, 8, 128, [4096] * 20, 4096, 0),            # 160 units > 148 SMs: balanced
    (16, 32, 8, 128, [9000] * 16, 4096, 2),            # clamped to the cache: still uniform
    (16, 32, 8, 128, [-5] * 8 + [4096] * 8, 4096, 0),  # negative lengths count as empty
    (36, 32, 8, 64, [3000] * 36, 3008, 0),             # 288 units
    (18, 16, 8, 64, [3000] * 18, 3008, 2),             # 144 units on 148 SMs (D = 64 uses every SM)
    (4, 40, 2, 64, [1500] * 4, 1536, 0),               # 16 units: balanced spreads them wider
    (1, 4, 1, 64, [256], 256, 2),                      # the tiny case: one unit, one launch
    (16, 32, 8, 32, [16384] * 16, 16384, 2),           # other head dims at 128 equal units
    (16, 32, 8, 64, [8192] * 16, 8192, 2),
    (16, 32, 8, 256, [2048] * 16, 2048, 2),
    (16, 64, 2, 128, [16384] * 16, 16384, 3),          # 32 q heads per kv head at D = 128: tensor cores
    (16, 64, 2, 64, [16384] * 16, 16384, 0),           # two head blocks per kv head: balanced, shared ring
])
def test_plan_cta_local_from_host_lengths(B, Hq, Hkv, D, lens, cap, want):
    pl = apd.query_plan(B, Hq, Hkv, D, 0, sm_count=148, host_seq_lens=lens, max_seq_len=cap)
    assert pl.mode == want
    assert (want == 2) == cta_local_expected(B, Hq, Hkv, D, lens, cap)
    if want == 2:
        units = B * Hkv * pl.head_blocks
        assert pl.grid_ctas == units and pl.num_workers == units * pl.warps_per_cta
        assert pl.combine_ctas == 0 and pl.partial_slots == 0
        assert pl.workspace_bytes <= apd.workspace_size(B, Hq, Hkv, D, 0)
    else:
        assert pl == apd.query_plan(B, Hq, Hkv, D, 0, sm_count=148)


def test_plan_host_lengths_do_not_change_fixed_splits():
    lens = [4096] * 16
    for splits in (1, 4):
        assert apd.query_plan(16, 32, 8, 128, splits, sm_count=148, host_seq_lens=lens, max_seq_len=4096) == \
            apd.query_plan(16, 32, 8, 128, splits, sm_count=148)


def test_plan_host_lengths_checked():
    with pytest.raises(ValueError):
        apd.query_plan(16, 32, 8, 128, 0, sm_count=148, host_seq_lens=[4096] * 15, max_seq_len=4096)
    p = apd._Plan()
    lens = (ctypes.c_int32 * 2)(10, 10)
    assert apd.lib().apd_query_plan_ex(2, 8, 2, 64, 0, ctypes.c_size_t(-1).value, 148, ctypes.cast(lens, ctypes.c_void_p),
                                       -1, ctypes.byref(p)) == ARG


def test_plan_workspace_too_small_for_fixed_splits():
    need = apd.workspace_size(16, 32, 8, 128, 4)
    with pytest.raises(apd.APDError) as e:
        apd.query_plan(16, 32, 8, 128, 4, workspace_bytes=need - 256, sm_count=148)
    assert e.value.status == WS


def test_binding_fails_loudly_without_the_library(monkeypatch):
    monkeypatch.setattr(apd, "_lib", None)
    monkeypatch.setattr(apd, "_LIB_PATH", os.path.join(ROOT, "no_such_library.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        apd.workspace_size(1, 4, 1, 64)


def test_binding_rejects_five_dim_tensors():
    with pytest.raises(ValueError):
        apd._desc(torch.zeros(1, 1, 1, 1, 1))


def test_empty_batch_accepts_null_batch_tensors():
    p = problem(B=0)
    for f in ("q", "pt", "sl", "out"):
        p[f].data = None
    assert call(p) == OK
    p = problem(B=0)
    p["k"].data = None
    assert call(p) == NULLP


# ---------------------------------------------------------------- contiguous KV
def contig_call(p, splits=0, ws=FAKE, ws_bytes=1 << 30):
    return apd.lib().apd_attn_contig_decode(ctypes.byref(p["q"]), ctypes.byref(p["k"]), ctypes.byref(p["v"]),
                                            ctypes.byref(p["sl"]), ctypes.byref(p["out"]), ctypes.c_float(0.1),
                                            splits, ws, ws_bytes, None)


def contig_problem(B=2, Hq=8, Hkv=2, D=64, Lmax=1000):
    return dict(q=T([B, Hq, D]), k=T([B, Lmax, Hkv, D]), v=T([B, Lmax, Hkv, D]), sl=T([B], apd.DTYPE_INT32),
                out=T([B, Hq, D]))


def test_contig_validation():
    # any Lmax is accepted (the call then needs a device, which this host does not have)
    assert contig_call(contig_problem(Lmax=1000)) in (OK, CUDA)
    assert contig_call(contig_problem(Lmax=7)) in (OK, CUDA)
    p = contig_problem()
    p["k"] = T([3, 1000, 2, 64])  # one KV row per sequence: leading extent must be B
    p["v"] = T([3, 1000, 2, 64])
    assert contig_call(p) == SHAPE
    assert contig_call(contig_problem(Hq=6, Hkv=4)) == GQA
    assert contig_call(contig_problem(D=96)) == HEADDIM
    assert contig_call(contig_problem(), splits=4, ws_bytes=1024) == WS
    p = contig_problem()
    p["k"].data = None
    assert contig_call(p) == NULLP
    assert contig_call(contig_problem(B=0)) == OK


def test_paged_entry_still_rejects_a_null_page_table_descriptor():
    p = problem()
    L = apd.lib()
    rc = L.apd_attn_paged_decode(ctypes.byref(p["q"]), ctypes.byref(p["k"]), ctypes.byref(p["v"]), None,
                                 ctypes.byref(p["sl"]), ctypes.byref(p["out"]), ctypes.c_float(1.0), 0, FAKE, 1 << 30,
                                 None)
    assert rc == NULLP
    rc = L.apd_attn_paged_decode_noalloc(ctypes.byref(p["q"]), ctypes.byref(p["k"]), ctypes.byref(p["v"]), None,
                                         ctypes.byref(p["sl"]), ctypes.byref(p["out"]), ctypes.c_float(1.0), 0, None)
    assert rc == NULLP


# ---------------------------------------------------------------- GEMV
def gemv_call(x, w, y, ws=FAKE, ws_bytes=1 << 30):
    return apd.lib().apd_gemv_bf16(ctypes.byref(x), ctypes.byref(w), ctypes.byref(y), ws, ws_bytes, None)


def test_gemv_validation():
    assert gemv_call(T([9, 64]), T([16, 64]), T([9, 16])) == SHAPE      # M > 8
    assert gemv_call(T([2, 64]), T([16, 32]), T([2, 16])) == SHAPE      # K mismatch
    assert gemv_call(T([2, 64]), T([16, 64]), T([2, 15])) == SHAPE      # y shape
    assert gemv_call(T([2, 60]), T([16, 60]), T([2, 16])) == LAYOUT     # K % 8
    assert gemv_call(T([2, 64], stride=[68, 1]), T([16, 64]), T([2, 16])) == LAYOUT  # row stride not 16-B
    assert gemv_call(T([2, 64], apd.DTYPE_FP32), T([16, 64]), T([2, 16])) == DTYPE
    x = T([2, 64]); x.data = None
    assert gemv_call(x, T([16, 64]), T([2, 16])) == NULLP
    assert gemv_call(T([2, 64]), T([16, 64]), T([2, 16]), ws=None) == WS
    assert apd.lib().apd_gemv_workspace_size(9, 16, 64) == 0
    assert apd.gemv_workspace_size(8, 100000, 1536) % 256 == 0


# ---------------------------------------------------------------- multi-query (prefill)
def prefill_call(p, kernel=0, causal=-1, mask=None):
    return apd.lib().apd_attn_paged_prefill_ex(
        ctypes.byref(p["q"]), ctypes.byref(p["k"]), ctypes.byref(p["v"]), ctypes.byref(p["pt"]),
        ctypes.byref(p["sl"]), ctypes.byref(mask) if mask is not None else None, ctypes.byref(p["out"]),
        ctypes.c_float(0.1), causal, None, kernel)


def prefill_problem(B=2, Lq=5, Hq=8, Hkv=2, D=64, P=32, NP=16, MP=4):
    return dict(q=T([B, Lq, Hq, D]), k=T([NP, P, Hkv, D]), v=T([NP, P, Hkv, D]),
                pt=T([B, MP], apd.DTYPE_INT32), sl=T([B], apd.DTYPE_INT32), out=T([B, Lq, Hq, D]))


def test_prefill_kernel_choice_is_validated_before_any_launch():
    for bad in (-1, 3, 99):
        assert prefill_call(prefill_problem(), kernel=bad) == ARG
    for k in apd.PREFILL_KERNELS.values():
        for D in (32, 64, 128, 256):  # every head dim on every kernel (the call then needs a device)
            assert prefill_call(prefill_problem(D=D), kernel=k) in (OK, CUDA)
        assert prefill_call(prefill_problem(D=96), kernel=k) == HEADDIM
        assert prefill_call(prefill_problem(B=0), kernel=k) == OK
        assert prefill_call(prefill_problem(Hq=6, Hkv=4), kernel=k) == GQA
        assert prefill_call(prefill_problem(), kernel=k, causal=-2) == ARG
    mask = T([2, 100], apd.DTYPE_UINT8)  # shorter than MP * P = 128
    assert prefill_call(prefill_problem(), mask=mask) == SHAPE


def test_prefill_binding_rejects_unknown_kernel_names():
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        apd.attn_paged_prefill(q, q, q, torch.zeros(1, 1, dtype=torch.int32), torch.zeros(1, dtype=torch.int32),
                               0.1, kernel="wgmma")


def test_selftest_arguments_are_checked_before_any_launch():
    L = apd.lib()
    assert L.apd_selftest_bounded_wait(None, 1000, None) == NULLP
    assert L.apd_selftest_bounded_wait(FAKE, 0, None) == ARG
    assert L.apd_selftest_bounded_wait(FAKE, 2_000_000_000, None) == ARG


def test_release_selftest_arguments_are_checked_before_any_launch():
    """The shared-ring release self-test: a NULL page table, a limit outside 1 ns .. 1 s, and a
    problem that does not take the shared ring (g <= 16) are refused without a launch."""
    L = apd.lib()

    def call(p, limit=1_000_000, pt=True):
        a = [ctypes.byref(p[n]) for n in ("q", "k", "v")] + [ctypes.byref(p["pt"]) if pt else None] + \
            [ctypes.byref(p[n]) for n in ("sl", "out")]
        return L.apd_selftest_shared_ring_release(*a, ctypes.c_float(0.1), FAKE, 1 << 30, limit, None)

    g32 = dict(q=T([2, 64, 128]), out=T([2, 64, 128]), k=T([16, 32, 2, 128]), v=T([16, 32, 2, 128]),
               pt=T([2, 4], apd.DTYPE_INT32), sl=T([2], apd.DTYPE_INT32))
    assert call(g32, pt=False) == NULLP
    assert call(g32, limit=0) == ARG
    assert call(g32, limit=2_000_000_000) == ARG
    g4 = dict(g32, q=T([2, 8, 128]), out=T([2, 8, 128]))
    assert call(g4) in (ARG, CUDA)  # ARG once the plan is made (it needs the device's SM count)


def test_stall_selftest_arguments_are_checked_before_any_launch():
    """The tensor-core kernel's stall self-test: a NULL page table, a limit outside 1 ns ..
    1 s, and a problem that does not take that kernel (g = 4) are refused without a launch."""
    L = apd.lib()

    def call(p, limit=1_000_000, pt=True):
        a = [ctypes.byref(p[n]) for n in ("q", "k", "v")] + [ctypes.byref(p["pt"]) if pt else None] + \
            [ctypes.byref(p[n]) for n in ("sl", "out")]
        return L.apd_selftest_mq_tc_stall(*a, ctypes.c_float(0.1), 0, FAKE, 1 << 30, limit, None)

    g32 = dict(q=T([2, 64, 128]), out=T([2, 64, 128]), k=T([16, 32, 2, 128]), v=T([16, 32, 2, 128]),
               pt=T([2, 4], apd.DTYPE_INT32), sl=T([2], apd.DTYPE_INT32))
    assert call(g32, pt=False) == NULLP
    assert call(g32, limit=0) == ARG
    assert call(g32, limit=2_000_000_000) == ARG
    g4 = dict(g32, q=T([2, 8, 128]), out=T([2, 8, 128]))
    assert call(g4) in (ARG, CUDA)  # ARG once the plan is made (it needs the device's SM count)


# ---------------------------------------------------------------- GEMV planning
@pytest.mark.parametrize("M,N,K", [(1, 100000, 1536), (8, 100000, 1536), (1, 6912, 1536), (3, 1536, 1536),
                                   (1, 256, 1536), (8, 1536, 6912), (5, 50, 1040), (2, 3000, 1000), (1, 64, 200),
                                   (4, 2048, 16384), (1, 2360, 520)])
def test_gemv_plan(M, N, K):
    _check_gemv_plan(M, N, K)


def _check_gemv_plan(M, N, K):
    p = apd.gemv_query_plan(M, N, K, 148)
    mtiles, ktiles = -(-N // 16), -(-K // 256)
    # x is staged once per CTA for weight streams of at least 64 MB when its padded rows
    # (16-byte chunks, an odd number per row) take at most 32 KB and fit beside the ring
    x_bytes = M * 16 * ((K // 8) | 1)
    xs = N * K * 2 >= (64 << 20) and x_bytes <= 32768 and 8 * 6 * 4 + 8 + 16 + x_bytes + 32 + 1024 + 6 * 4 * 8192 <= 232448
    assert p["x_staged"] == int(xs)
    # short weight streams with fewer 16-row tiles than SMs: one CTA per tile, up to 4
    # warps splitting its k-tiles, parts added in shared memory, one kernel
    cta = not xs and mtiles <= 148 and ktiles >= 2 and N * K * 2 <= (32 << 20)
    assert p["cta_per_mtile"] == int(cta)
    if cta:
        assert p["warps_per_cta"] == min(4, ktiles) and p["grid_ctas"] == mtiles
        assert p["workers"] == mtiles * p["warps_per_cta"] and p["sum_ctas"] == 0
        assert p["workspace_bytes"] == 256
        return
    assert p["stages"] == 4
    whole = mtiles >= 148 and mtiles <= 148 * (6 if xs else 4) and ktiles <= 8
    if whole:
        # one warp per m-tile, as few warps per CTA as put every SM to work
        assert p["warps_per_cta"] == min(6 if xs else 4, -(-mtiles // 148))
        assert p["workers"] == mtiles and p["sum_ctas"] == 0
    else:
        assert p["warps_per_cta"] == (6 if xs else 4)
        assert p["workers"] == min(148 * (7 if xs else 8) // 8 * p["warps_per_cta"], mtiles * ktiles)
        assert p["sum_ctas"] == -(-mtiles // 4)
    assert p["grid_ctas"] == -(-p["workers"] // p["warps_per_cta"])
    assert p["workspace_bytes"] == 256 + -(-(2 * p["workers"] * 16 * 8 * 4) // 256) * 256


@settings(max_examples=300, deadline=None)
@given(M=st.integers(1, 8), N=st.integers(1, 200000), K8=st.integers(1, 2048))
def test_gemv_plan_random_shapes(M, N, K8):
    """The restated GEMV launch rule over random shapes (K a multiple of 8, as the call
    requires)."""
    _check_gemv_plan(M, N, 8 * K8)


def test_gemv_plan_rejects_bad_shapes():
    for m, n, k in ((0, 16, 64), (9, 16, 64), (1, 0, 64), (1, 16, 0)):
        with pytest.raises(apd.APDError):
            apd.gemv_query_plan(m, n, k, 148)


# ---------------------------------------------------------------- plan invariants


@settings(max_examples=300, deadline=None)
@given(B=st.integers(1, 300), Hkv=st.sampled_from([1, 2, 4, 8, 16]), g=st.integers(1, 200),
       D=st.sampled_from([32, 64, 128, 256]), sm=st.sampled_from([1, 8, 132, 148]),
       splits=st.sampled_from([0, 0, 1, 3]), L=st.integers(0, 70000))
def test_plan_invariants(B, Hkv, g, D, sm, splits, L):
    """Whatever the shape, SM count or hint, a plan is one the kernels can run:
    - its shared memory fits a CTA;
    - every CTA's warps are within the launch bound;
    - the grid covers the workers;
    - with a shared K/V ring, the head blocks of a kv head share a CTA;
    - with fixed splits, one unit-kernel CTA per split of each unit;
    - with the one-CTA-per-unit plan, each unit gets its own SM and no combine runs."""
    Hq = Hkv * g
    hb = -(-g // 16)
    pl = apd.query_plan(B, Hq, Hkv, D, splits, sm_count=sm, host_seq_lens=[L] * B, max_seq_len=70000)
    bound = {32: 16, 64: 10}.get(D, 8) if not pl.shared_kv_ring else 8
    if pl.mode == 3:
        bound = 11  # the tensor-core kernel at 64 heads: 2 softmax groups + 3 warps
    assert pl.smem_bytes <= 232448
    assert 1 <= pl.warps_per_cta <= bound
    assert pl.grid_ctas * pl.warps_per_cta >= pl.num_workers > 0
    assert pl.head_blocks == hb and pl.rows_per_unit == min(g, 16)
    units = B * Hkv * hb
    if pl.shared_kv_ring:
        assert pl.mode == 0 and hb > 1 and D != 32
        assert pl.warps_per_cta % hb == 0 and pl.num_workers % (Hkv * hb) == 0
    if pl.mode == 0:
        # at most one CTA per SM, unless one worker group alone needs more CTAs (the CTAs
        # never wait on one another, so they may also run in waves)
        assert splits == 0 and pl.num_workers % (Hkv * hb) == 0
        assert pl.grid_ctas <= max(sm, -(-(Hkv * hb) // pl.warps_per_cta))
    elif pl.mode == 1:
        assert splits > 0 and pl.grid_ctas == units * splits
        assert pl.num_workers == pl.grid_ctas * pl.warps_per_cta
    elif pl.mode == 3:
        # the tensor-core multi-query kernel: one CTA per split of each (sequence, kv head,
        # block of at most 64 q heads)
        nb = -(-g // 64)
        assert D == 128 and g > 16 and pl.q_head_blocks == nb and pl.grid_ctas % (B * Hkv * nb) == 0
        assert pl.q_heads_per_block % 16 == 0 and pl.q_heads_per_block <= 64
        assert (nb - 1) * pl.q_heads_per_block < g <= nb * pl.q_heads_per_block
        k = pl.grid_ctas // (B * Hkv * nb)
        assert k == splits or splits == 0
        assert pl.partial_slots == (units * k if k > 1 else 0)
        assert pl.cluster_size in (0, k) and (pl.cluster_size == 0 or 2 <= k <= 8)
        assert (pl.combine_ctas == 0) == (k == 1 or pl.cluster_size > 0)
    else:
        assert splits == 0 and pl.mode == 2 and units <= sm
        assert pl.grid_ctas == units and pl.combine_ctas == 0 and pl.partial_slots == 0
