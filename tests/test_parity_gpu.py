"""GPU parity: the CUDA path (through the C-ABI binding) against the fp64 CPU oracle.

Every comparison is element by element on the same seeded inputs, with the
per-element bound |gpu - ref| <= 1e-2 + 1e-2 |ref| (ref = fp64 oracle value).
Covered: the tiny decode case, the full head-dim / GQA / split sweep, HND
storage, NaN-poisoned slots that must never be read, ragged and empty
sequences, head groups that span several 16-row blocks, larger pages, strided
q / out, a side stream, CUDA-graph capture, determinism, the device-side
contract flags, and the three large decode workloads at full size in the launch
configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads
from gpu_util import DeviceProblem, check_close

pytestmark = pytest.mark.gpu


def small(seed, B, Hq, Hkv, D, lens, P=32, pool=None, **kw):
    return workloads.make(name="case", seed=seed, batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          page_size=P, seq_lens=list(lens), pool_pages=pool, **kw)


# ---------------------------------------------------------------- named small workloads
@pytest.mark.parametrize("splits", [1, 0, 4, 8])
def test_tiny(splits):
    w = workloads.tiny()
    ref = oracle.paged_decode(w)
    check_close(DeviceProblem(w).run(splits), ref, f"tiny splits={splits}")


@pytest.mark.parametrize("D,Hq,Hkv,S", list(workloads.sweep_cases()))
def test_sweep(D, Hq, Hkv, S):
    w = workloads.sweep_case(D, Hq, Hkv, S)
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    check_close(dp.run(S), ref, w.name)
    check_close(dp.run(0), ref, w.name + " auto")


@pytest.mark.parametrize("D", workloads.SWEEP_HEAD_DIMS)
@pytest.mark.parametrize("S", [1, 3, 0])
def test_sweep_hnd_layout(D, S):
    w = workloads.sweep_case(D, 32, 8, S, layout="HND", seed=99)
    assert w.k_cache.stride(2) != D  # really strided
    check_close(DeviceProblem(w).run(S), oracle.paged_decode(w), f"HND D={D} S={S}")


@pytest.mark.parametrize("D", workloads.SWEEP_HEAD_DIMS)
@pytest.mark.parametrize("S", [1, 4, 0])
def test_poisoned_slots_are_never_read(D, S):
    """Tail slots, unused pool pages and unused page-table entries hold NaN."""
    w = small(7, B=5, Hq=16, Hkv=4, D=D, lens=(1, 31, 33, 200, 515), pool=40, poison=True,
              max_pages_per_seq=20)
    ref = oracle.paged_decode(w)
    assert np.isfinite(ref).all()
    check_close(DeviceProblem(w).run(S), ref, f"poison D={D} S={S}")


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [1, 3, 0, 148])
def test_ragged_and_empty_sequences(D, S):
    lens = (0, 1, 31, 32, 33, 64, 65, 1000, 0, 7)
    w = small(21, B=len(lens), Hq=8, Hkv=2, D=D, lens=lens, pool=60, poison=True, max_pages_per_seq=32)
    ref = oracle.paged_decode(w)
    out = DeviceProblem(w).run(S)
    check_close(out, ref, f"ragged D={D} S={S}")
    assert torch.all(out[0] == 0) and torch.all(out[8] == 0)


@pytest.mark.parametrize("S", [0, 3])
def test_large_batch_combine_walks_the_units(S):
    """Batches with more units than the combine grid (at most 4 CTAs per SM): its CTAs walk
    several units each, skipping the units one warp covered and writing the zero rows of
    empty sequences (auto splits), or merging fixed splits."""
    rng = np.random.default_rng(5)
    lens = rng.integers(0, 400, size=700)
    lens[::37] = 0
    w = small(23, B=700, Hq=8, Hkv=1, D=64, lens=lens, pool=int(sum((lens + 31) // 32)) + 8, poison=True,
              max_pages_per_seq=13)
    pl = apd.query_plan(700, 8, 1, 64, S)
    assert 0 < pl.combine_ctas < 700  # units per combine CTA > 1
    out = DeviceProblem(w).run(S)
    check_close(out, oracle.paged_decode(w), f"large batch S={S}")
    assert torch.all(out[torch.from_numpy(lens == 0).to(out.device)] == 0)


@pytest.mark.parametrize("S", [1, 0, 5])
def test_all_sequences_empty(S):
    w = small(22, B=3, Hq=4, Hkv=1, D=64, lens=(0, 0, 0), pool=2, max_pages_per_seq=4)
    out = DeviceProblem(w).run(S)
    assert torch.all(out == 0)


@pytest.mark.parametrize("D", [64, 128])
def test_empty_sequence_when_one_group_covers_every_position(D):
    """At most one tile per unit: a single worker group, no combine kernel; the
    empty sequence's rows are still written (zeros)."""
    w = small(24, B=1, Hq=8, Hkv=2, D=D, lens=(0,), P=32, pool=2, max_pages_per_seq=1)
    out = DeviceProblem(w).run(0)
    assert torch.all(out == 0)


def test_small_workspace_one_group_with_empty_sequences():
    """A workspace with room for one worker group only: every unit runs unsplit in
    one launch, and empty sequences still come out as zeros."""
    lens = (0, 100, 0, 37, 0)
    w = small(25, B=len(lens), Hq=8, Hkv=2, D=64, lens=lens, pool=12, max_pages_per_seq=4)
    dims = (w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim)
    lo, hi = 256, apd.workspace_size(*dims, 0)
    while lo < hi:  # the smallest workspace the balanced plan accepts
        mid = (lo + hi) // 512 * 256
        try:
            apd.query_plan(*dims, 0, workspace_bytes=mid)
            hi = mid
        except apd.APDError:
            lo = mid + 256
    plan = apd.query_plan(*dims, 0, workspace_bytes=hi)
    assert plan.num_workers == w.num_kv_heads and plan.combine_ctas == 0
    ws = torch.zeros(hi, dtype=torch.uint8, device="cuda")
    out = DeviceProblem(w).run(0, workspace=ws)
    check_close(out, oracle.paged_decode(w), "one group, small workspace")
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0) and torch.all(out[4] == 0)


def test_empty_batch():
    w = small(23, B=1, Hq=4, Hkv=1, D=64, lens=(5,), pool=2)
    dp = DeviceProblem(w)
    q0 = dp.q[:0]
    out0 = dp.out[:0]
    ws = apd.alloc_workspace(0 + 1, 4, 1, 64, 0)
    apd.attn_paged_decode(q0, dp.k, dp.v, dp.page_table[:0], dp.seq_lens[:0], out0, w.scale, 0, ws)


@pytest.mark.parametrize("Hq,Hkv", [(12, 4), (40, 2), (64, 2), (16, 1), (7, 7), (48, 1)])
@pytest.mark.parametrize("S", [1, 0, 4])
def test_gqa_groups(Hq, Hkv, S):
    """g = 3, 20 (a partial second 16-row head block), 32, 16, 1, 48."""
    w = small(31, B=3, Hq=Hq, Hkv=Hkv, D=64, lens=(45, 300, 129), pool=30)
    check_close(DeviceProblem(w).run(S), oracle.paged_decode(w), f"gqa {Hq}/{Hkv} S={S}")


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("Hq,Hkv", [(40, 2), (64, 2), (48, 1), (80, 1)])
@pytest.mark.parametrize("ws_div", [1, 16])
def test_shared_kv_ring(D, Hq, Hkv, ws_div):
    """Balanced mode with g = 20, 32, 48, 80 (2 to 5 head blocks per kv head): the head
    blocks of a kv head read one K/V ring (except D = 32, D = 256 with 5 head blocks, and
    D = 128, which takes the tensor-core multi-query kernel).  Ragged lengths with an empty
    sequence and a partial last tile, NaN-poisoned unused slots; ws_div = 16 gives a workspace a sixteenth
    of the default, so fewer groups and runs of many tiles per warp (every stage's release
    barrier goes through many phases)."""
    lens = (1500, 0, 33, 777)
    w = small(71, B=4, Hq=Hq, Hkv=Hkv, D=D, lens=lens, pool=90, poison=True)
    dp = DeviceProblem(w)
    default = apd.workspace_size(4, Hq, Hkv, D, 0)
    ws = torch.zeros(default // ws_div // 256 * 256, dtype=torch.uint8, device="cuda")  # flags start clear
    pl = apd.query_plan(4, Hq, Hkv, D, 0, workspace_bytes=ws.numel())
    # D = 32 keeps one ring per warp; D = 256 takes at most 4 warps per CTA, so 5 head
    # blocks keep one ring per warp too
    shared = D != 32 and not (D == 256 and pl.head_blocks > 4)
    if D == 128:
        assert pl.mode == 3  # the tensor-core multi-query kernel (tests/test_mq_tc_gpu.py)
    else:
        assert pl.mode == 0 and pl.shared_kv_ring == int(shared)
        assert pl.warps_per_cta % pl.head_blocks == 0 or not shared
    check_close(dp.run(0, workspace=ws), oracle.paged_decode(w), f"shared ring D={D} {Hq}/{Hkv} ws/{ws_div}")
    assert apd.read_device_flags(ws) == 0


@pytest.mark.parametrize("D,Hq,Hkv", [(64, 160, 2), (64, 48, 1), (256, 96, 2)])
def test_shared_kv_ring_one_group(D, Hq, Hkv):
    """The shared K/V ring with a workspace that holds one worker group only: every warp
    streams all positions, units are written directly (no combine kernel), and the
    workers write the zero rows of the empty sequences.  Pages of 64 tokens put two tiles
    in a page, so the page-slot cursor steps within pages too."""
    lens = (0, 700, 0, 65, 1)
    w = small(73, B=len(lens), Hq=Hq, Hkv=Hkv, D=D, lens=lens, P=64, pool=20, poison=True,
              max_pages_per_seq=12)
    dims = (w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim)
    lo, hi = 256, apd.workspace_size(*dims, 0)
    while lo < hi:  # the smallest workspace the balanced plan accepts
        mid = (lo + hi) // 512 * 256
        try:
            apd.query_plan(*dims, 0, workspace_bytes=mid)
            hi = mid
        except apd.APDError:
            lo = mid + 256
    plan = apd.query_plan(*dims, 0, workspace_bytes=hi)
    hb = -(-(Hq // Hkv) // 16)
    assert plan.shared_kv_ring == 1 and plan.num_workers == Hkv * hb and plan.combine_ctas == 0
    ws = torch.zeros(hi, dtype=torch.uint8, device="cuda")
    out = DeviceProblem(w).run(0, workspace=ws)
    check_close(out, oracle.paged_decode(w), f"shared ring, one group, D={D} {Hq}/{Hkv}")
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    assert apd.read_device_flags(ws) == 0


@pytest.mark.parametrize("P", [64, 128])
@pytest.mark.parametrize("S", [1, 0, 3])
def test_larger_pages(P, S):
    w = small(41, B=4, Hq=8, Hkv=2, D=128, lens=(1, 100, 257, 640), P=P, pool=24, poison=True,
              max_pages_per_seq=12)
    check_close(DeviceProblem(w).run(S), oracle.paged_decode(w), f"P={P} S={S}")


@pytest.mark.parametrize("D", [32, 256])
def test_max_head_dim_and_group(D):
    """D extremes with a full 16-row head block and a long sequence."""
    w = small(43, B=2, Hq=32, Hkv=2, D=D, lens=(2049, 77), pool=70)
    for S in (1, 0, 16):
        check_close(DeviceProblem(w).run(S), oracle.paged_decode(w), f"D={D} S={S}")


def test_strided_q_and_out():
    w = small(51, B=3, Hq=8, Hkv=2, D=64, lens=(40, 90, 3), pool=8)
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    big_q = torch.zeros(3, 8, 192, dtype=torch.bfloat16, device="cuda")
    big_q[:, :, 64:128] = dp.q
    q = big_q[:, :, 64:128]
    big_out = torch.full((3, 10, 72), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = big_out[:, 1:9, 8:]
    ws = apd.alloc_workspace(3, 8, 2, 64, 0)
    apd.attn_paged_decode(q, dp.k, dp.v, dp.page_table, dp.seq_lens, out, w.scale, 0, ws)
    check_close(out, ref, "strided")
    assert torch.isnan(big_out[:, 0]).all() and torch.isnan(big_out[:, 9]).all()
    assert torch.isnan(big_out[:, :, :8]).all()


def test_side_stream():
    w = small(52, B=4, Hq=16, Hkv=4, D=128, lens=(500, 20, 1, 900), pool=50)
    dp = DeviceProblem(w)
    s = torch.cuda.Stream()
    ws = apd.alloc_workspace(4, 16, 4, 128, 0)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws)
    s.synchronize()
    check_close(dp.out, oracle.paged_decode(w), "side stream")


@pytest.mark.parametrize("S", [0, 1, 4])
def test_cuda_graph_capture_and_replay(S):
    w = small(53, B=4, Hq=32, Hkv=8, D=128, lens=(300, 1, 77, 1024), pool=60)
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(4, 32, 8, 128, S)
    eager = dp.run(S, workspace=ws).clone()
    out = torch.full_like(dp.out, float("nan"))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, out, w.scale, S, ws)  # live first
        with torch.cuda.graph(g, stream=s):
            apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, out, w.scale, S, ws)
    torch.cuda.current_stream().wait_stream(s)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    # new inputs in the same buffers are picked up by the replay
    dp.q.mul_(-1)
    g.replay()
    torch.cuda.synchronize()
    w.q.mul_(-1)
    check_close(out, oracle.paged_decode(w), "graph replay with new q")


def test_split_done_event_inside_a_graph_times_the_split_kernel():
    """Recorded while the stream is captured, the split-done event becomes an event-record
    node: each replay stamps it between the two kernels, and the result is unchanged."""
    w = small(54, B=4, Hq=32, Hkv=8, D=128, lens=(3000, 1, 777, 4096), pool=300)
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(4, 32, 8, 128, 0)
    eager = dp.run(0, workspace=ws).clone()
    b = torch.cuda.Event(enable_timing=True, external=True)
    m = torch.cuda.Event(enable_timing=True, external=True)
    e = torch.cuda.Event(enable_timing=True, external=True)
    s = torch.cuda.Stream()
    for ev in (b, m, e):
        ev.record(s)
    s.synchronize()
    out = torch.full_like(dp.out, float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            b.record(s)
            apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, out, w.scale, 0, ws, stream=s,
                                  split_done_event=m)
            e.record(s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    split_ms, call_ms = b.elapsed_time(m), b.elapsed_time(e)
    assert 0 < split_ms <= call_ms, (split_ms, call_ms)


def test_inputs_written_by_the_preceding_kernel_are_seen():
    """The split kernel may start launching before the previous kernel in the stream
    ends (programmatic dependent launch); it must still read q, page_table and
    seq_lens only after that kernel's writes.  Each call here follows torch kernels
    that rewrite those inputs in place."""
    ws_len = (700, 64, 1500)
    w = small(54, B=3, Hq=16, Hkv=4, D=128, lens=ws_len, pool=80, max_pages_per_seq=48)
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(3, 16, 4, 128, 0)
    call = apd.DecodeCall(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws)
    qs = [torch.randn(3, 16, 128, generator=torch.Generator().manual_seed(i)).to(torch.bfloat16) for i in range(4)]
    lens = [torch.tensor(x, dtype=torch.int32) for x in ((700, 64, 1500), (1, 1200, 33), (0, 1536, 640), (95, 5, 1))]
    outs = []
    qs_dev = [q.cuda() for q in qs]
    lens_dev = [l.cuda() for l in lens]
    for i in range(4):
        dp.q.copy_(qs_dev[i])
        dp.seq_lens.copy_(lens_dev[i])
        call()
        outs.append(dp.out.clone())
    torch.cuda.synchronize()
    for i in range(4):
        w.q.copy_(qs[i])
        w.seq_lens.copy_(lens[i])
        check_close(outs[i], oracle.paged_decode(w), f"step {i}")


@pytest.mark.parametrize("S", [0, 1, 4])
def test_deterministic(S):
    """Auto splits without the host-length hint (balanced plan) and fixed splits give the
    same bits on every call."""
    w = workloads.sweep_case(128, 32, 8, S)
    dp = DeviceProblem(w)
    a = dp.run(S).clone()
    b = dp.run(S).clone()
    assert torch.equal(a, b)


def test_one_cta_per_unit_repeats_within_tolerance():
    """With the host-length hint the one-CTA-per-unit plan lets warps take tiles in the order
    they become free, so calls may differ in the last bits: each one still matches the
    oracle, and two calls differ by far less than that tolerance: the parts weight their
    bf16 probabilities against different running maxima, so the difference is bf16 rounding
    noise of the weights, of order 1e-4 in absolute terms."""
    w = workloads.llama8b()
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(16, 32, 8, 128, 0)
    call = apd.DecodeCall(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws,
                          host_seq_lens=w.seq_lens)
    pl = apd.query_plan(16, 32, 8, 128, 0, host_seq_lens=w.seq_lens, max_seq_len=w.page_table.shape[1] * 32)
    assert pl.mode == 2
    ref = oracle.paged_decode(w)
    outs = []
    for _ in range(3):
        call()
        outs.append(dp.out.clone())
        check_close(outs[-1], ref, "one CTA per unit")
    a, b = outs[0].float(), outs[1].float()
    assert ((a - b).abs() <= 2e-3 + 2.0 ** -6 * torch.maximum(a.abs(), b.abs())).all()


# ---------------------------------------------------------------- device-side contract
def test_out_of_range_pages_set_a_flag_and_read_zeros():
    w = small(61, B=3, Hq=8, Hkv=2, D=64, lens=(64, 64, 40), pool=8)
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    dp.page_table[1, 0] = w.num_pages + 3
    dp.page_table[1, 1] = -2
    ws = apd.alloc_workspace(3, 8, 2, 64, 0)
    apd.workspace_init(ws)
    apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws)
    flags = apd.read_device_flags(ws)
    assert flags & apd.FLAG_PAGE_OUT_OF_RANGE
    out = dp.out.to(torch.float64).cpu().numpy()
    assert np.isfinite(out).all()
    # sequence 1 read only zero rows: every weight equal, V rows zero -> output 0
    assert np.all(out[1] == 0)
    check_close(dp.out[[0, 2]], ref[[0, 2]], "untouched sequences")
    assert apd.read_device_flags(ws) == 0  # cleared by the previous read


def test_seq_len_contract_flags():
    w = small(62, B=3, Hq=4, Hkv=1, D=64, lens=(64, 10, 20), pool=6, max_pages_per_seq=2)
    dp = DeviceProblem(w)
    dp.seq_lens[1] = 5000   # > max_pages * page_size = 64: clamped to 64
    dp.seq_lens[2] = -7     # treated as 0
    ws = apd.alloc_workspace(3, 4, 1, 64, 0)
    apd.workspace_init(ws)
    apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws)
    flags = apd.read_device_flags(ws)
    assert flags & apd.FLAG_SEQ_LEN_CLAMPED and flags & apd.FLAG_SEQ_LEN_NEGATIVE
    assert not flags & apd.FLAG_PAGE_OUT_OF_RANGE
    assert torch.all(dp.out[2] == 0)
    w.seq_lens[1] = 64
    w.seq_lens[2] = 0
    check_close(dp.out, oracle.paged_decode(w), "clamped lengths")


def test_bad_arguments_raise_before_launch():
    w = small(63, B=2, Hq=8, Hkv=2, D=64, lens=(10, 20), pool=2)
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(2, 8, 2, 64, 4)
    with pytest.raises(apd.APDError) as e:
        apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 4, ws[:1024])
    assert e.value.status == 9
    with pytest.raises(apd.APDError) as e:
        apd.attn_paged_decode(dp.q.float(), dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws)
    assert e.value.status == 2


# ---------------------------------------------------------------- full-size workloads
@pytest.fixture(scope="module")
def llama():
    w = workloads.llama8b()
    return w, oracle.paged_decode(w)


@pytest.mark.parametrize("S", [0, 1, 4, 148])
def test_llama8b_full_size(llama, S):
    w, ref = llama
    check_close(DeviceProblem(w).run(S), ref, f"llama8b S={S}")


@pytest.mark.parametrize("S", [0, 148])
def test_long_context_full_size(S):
    w = workloads.long_context()
    ref = oracle.paged_decode(w)
    check_close(DeviceProblem(w).run(S), ref, f"long S={S}")


def test_ragged_full_size():
    w = workloads.ragged()
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    check_close(dp.run(0), ref, "ragged auto")
    check_close(dp.run(16), ref, "ragged S=16")


def test_llama8b_full_size_host_hint(llama):
    """The benchmark's launch: the host lengths select one CTA per (sequence, kv head),
    four parts merged in shared memory, one kernel."""
    w, ref = llama
    lens = w.seq_lens.tolist()
    assert apd.query_plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, 0, host_seq_lens=lens,
                          max_seq_len=w.page_table.shape[1] * w.page_size).mode == 2
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, 0)
    apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws, host_seq_lens=lens)
    check_close(dp.out, ref, "llama8b host hint")
    assert apd.read_device_flags(ws) == 0


# ---------------------------------------------------------------- host-length hint (CTA-local plan)
def run_hinted(w, hint, stream=None):
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, 0)
    if dp.contig:
        apd.attn_contig_decode(dp.q, dp.k, dp.v, dp.seq_lens, dp.out, w.scale, 0, ws, stream=stream,
                               host_seq_lens=hint)
    else:
        apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws, stream=stream,
                              host_seq_lens=hint)
    return dp.out, ws


# Per head dim, a length whose tiles fit the CTA-local slack (1024 / D tiles) for every
# head shape below and cut into all, or all but one, of the CTA's warps (a ragged last tile
# included): 36 tiles in 12 parts at D = 32, 18 in 9 of 10 warps at D = 64.
HINT_LEN = {32: 1140, 64: 564, 128: 250, 256: 120}


@pytest.mark.parametrize("D", workloads.SWEEP_HEAD_DIMS)
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (40, 2), (8, 8), (48, 1)])
def test_host_hint_cta_local_matches_oracle(D, Hq, Hkv):
    """Equal lengths: the hint selects the one-kernel plan (mode 2) for g = 4 and 1; with
    more than one head block per kv head (g = 20, the second block partial, and 48) each
    block's CTA would stream the K/V again, so the balanced plan stays, or, at D = 128, the
    tensor-core multi-query kernel runs (mode 3)."""
    L = HINT_LEN[D]
    lens = [L] * 5
    mp = -(-L // 32)
    w = small(71, B=5, Hq=Hq, Hkv=Hkv, D=D, lens=lens, pool=5 * mp + 4, poison=True, max_pages_per_seq=mp)
    pl = apd.query_plan(5, Hq, Hkv, D, 0, host_seq_lens=lens, max_seq_len=mp * 32)
    if Hq // Hkv <= 16:
        assert pl.mode == 2 and pl.combine_ctas == 0
    else:
        assert pl.mode == (3 if D == 128 else 0)
    out, ws = run_hinted(w, lens)
    check_close(out, oracle.paged_decode(w), f"hint D={D} {Hq}/{Hkv}")
    assert apd.read_device_flags(ws) == 0


@pytest.mark.parametrize("D", [64, 128])
def test_host_hint_that_disagrees_with_the_device_lengths(D):
    """The hint promises equal short lengths; the device lengths are ragged, empty and
    long.  The plan follows the hint (mode 2), the result follows the device lengths."""
    lens = (0, 1, 1000, 31, 257, 0, 640)
    w = small(72, B=len(lens), Hq=16, Hkv=4, D=D, lens=lens, pool=80, poison=True, max_pages_per_seq=32)
    hint = [HINT_LEN[D]] * len(lens)
    assert apd.query_plan(len(lens), 16, 4, D, 0, host_seq_lens=hint, max_seq_len=32 * 32).mode == 2
    out, ws = run_hinted(w, hint)
    check_close(out, oracle.paged_decode(w), f"lying hint D={D}")
    assert torch.all(out[0] == 0) and torch.all(out[5] == 0)


def test_host_hint_contig_and_graph_replay():
    lens = [250] * 6
    w = workloads.make_contig(name="hint", seed=73, batch=6, num_q_heads=32, num_kv_heads=8, head_dim=128,
                              seq_lens=lens, lmax=256, layout="bhld")
    ref = oracle.paged_decode(w)
    out, _ = run_hinted(w, lens)
    check_close(out, ref, "contig hint")
    # the same call captured in a graph (the plan is baked in at capture) and replayed
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(6, 32, 8, 128, 0)
    call = apd.DecodeCall(dp.q, dp.k, dp.v, None, dp.seq_lens, dp.out, w.scale, 0, ws, host_seq_lens=lens)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        call(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            call(s)
    dp.out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    check_close(dp.out, ref, "contig hint graph")
