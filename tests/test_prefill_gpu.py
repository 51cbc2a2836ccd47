"""GPU parity of the multi-query (chunked prefill) call against the fp64 oracle.

Per element |gpu - ref| <= 1e-2 + 1e-2 |ref|, as for decode.  Covered: every head
dim, GQA groups 1/4/8/20, query counts from 1 to 70 (several 64-row blocks and a
ragged last block), no causal mask, causal offsets that cut the key range, 2-D and
3-D masks, rows that see no key (zeros), NaN-poisoned slots that must not be read,
larger pages, HND storage and a graph capture."""
import numpy as np
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads
from gpu_util import check_close

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["mma_sync", "tcgen05"])
def kernel(request):
    """Every case runs on both kernels."""
    return request.param


def run(w, stream=None, kernel="auto"):
    heads_outer = w.k_cache.stride(1) < w.k_cache.stride(2)  # HND storage passed as a view
    def dev(t):
        if heads_outer:
            return t.permute(0, 2, 1, 3).contiguous().cuda().permute(0, 2, 1, 3)
        return t.contiguous().cuda()
    q = w.q.cuda()
    mask = w.mask.cuda() if w.mask is not None else None
    out = torch.full_like(q, float("nan"))
    apd.attn_paged_prefill(q, dev(w.k_cache), dev(w.v_cache), w.page_table.cuda(), w.seq_lens.cuda(), w.scale,
                           w.causal_offset, mask, out, stream=stream, kernel=kernel)
    torch.cuda.synchronize()
    return out


def case(seed, D=64, Hq=8, Hkv=2, Lq=5, lens=(40, 9, 100), causal=-1, mask=None, P=32, **kw):
    mp = max(1, -(-max(lens) // P))
    return workloads.make_prefill(name="pf", seed=seed, batch=len(lens), q_len=Lq, num_q_heads=Hq,
                                  num_kv_heads=Hkv, head_dim=D, seq_lens=list(lens), page_size=P, causal_offset=causal,
                                  mask=mask, max_pages_per_seq=mp, **kw)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("causal", [-1, 60])
@pytest.mark.parametrize("mask", [None, "2d", "3d"])
@pytest.mark.parametrize("Lq", [5, 45])
def test_prefill_head_dims_causal_masks(D, causal, mask, Lq, kernel):
    """Lq = 5 gives 20 rows per kv head (one 128-row tile), Lq = 45 gives 180 rows
    (the two-tile tensor-core kernel for D = 64 and 128, second tile partly empty)."""
    w = case(3, D=D, Lq=Lq, causal=causal, mask=mask, poison=True)
    check_close(run(w, kernel=kernel), oracle.paged_prefill(w), f"D={D} Lq={Lq} causal={causal} mask={mask}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (32, 8), (64, 8), (40, 2)])
@pytest.mark.parametrize("Lq", [1, 16, 17, 70])
def test_prefill_groups_and_query_counts(D, Hq, Hkv, Lq, kernel):
    """Rows per kv head from 1 to 1400: one tile, two tiles, several CTAs per head and a
    ragged last CTA; g = 20 packs queries unevenly into the 128-row tiles."""
    w = case(5, D=D, Hq=Hq, Hkv=Hkv, Lq=Lq, lens=(300, 77), causal=300 - Lq)
    check_close(run(w, kernel=kernel), oracle.paged_prefill(w), f"D={D} {Hq}/{Hkv} Lq={Lq}")


def test_prefill_rows_that_see_nothing_are_zero(kernel):
    w = case(6, D=64, Lq=4, lens=(50, 0, 20), mask="3d", mask_keep=0.5)
    w.mask[0, 2] = 0  # query 2 of sequence 0 sees no key
    out = run(w, kernel=kernel)
    ref = oracle.paged_prefill(w)
    check_close(out, ref, "zero rows")
    assert torch.all(out[1] == 0) and torch.all(out[0, 2] == 0)


def test_prefill_causal_offset_zero(kernel):
    w = case(7, D=128, Lq=33, lens=(40, 100), causal=0, poison=True)
    check_close(run(w, kernel=kernel), oracle.paged_prefill(w), "causal 0")


@pytest.mark.parametrize("P", [64, 128])
def test_prefill_larger_pages_hnd(P, kernel):
    w = case(8, D=128, Hq=16, Hkv=4, Lq=9, lens=(257, 31), causal=250, P=P, layout="HND", poison=True)
    check_close(run(w, kernel=kernel), oracle.paged_prefill(w), f"P={P} HND")


def test_prefill_side_stream_and_graph(kernel):
    w = case(9, D=64, Hq=32, Hkv=8, Lq=12, lens=(200, 500), causal=480, mask="2d")
    q = w.q.cuda()
    k, v, pt, sl = w.k_cache.cuda(), w.v_cache.cuda(), w.page_table.cuda(), w.seq_lens.cuda()
    mask = w.mask.cuda()
    out = torch.empty_like(q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        apd.attn_paged_prefill(q, k, v, pt, sl, w.scale, w.causal_offset, mask, out, stream=s, kernel=kernel)
        with torch.cuda.graph(g, stream=s):
            apd.attn_paged_prefill(q, k, v, pt, sl, w.scale, w.causal_offset, mask, out, stream=s, kernel=kernel)
    torch.cuda.current_stream().wait_stream(s)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    check_close(out, oracle.paged_prefill(w), "graph replay")


def test_prefill_chunk_at_scale(kernel):
    """A 128-token chunk of 4 sequences of 1024 keys, 32/8 heads, D = 128, causal."""
    w = case(10, D=128, Hq=32, Hkv=8, Lq=128, lens=(1024, 1024, 1000, 640), causal=None or 0)
    w.causal_offset = 1024 - 128
    check_close(run(w, kernel=kernel), oracle.paged_prefill(w), "chunk at scale")


def test_prefill_rejects_bad_arguments():
    w = case(11, D=64, Lq=3, lens=(10, 20, 30), mask="2d")
    q = w.q.cuda()
    args = (w.k_cache.cuda(), w.v_cache.cuda(), w.page_table.cuda(), w.seq_lens.cuda(), w.scale)
    with pytest.raises(apd.APDError):  # causal offset below -1
        apd.attn_paged_prefill(q, *args, causal_offset=-5)
    with pytest.raises(apd.APDError):  # mask shorter than the page-table capacity
        apd.attn_paged_prefill(q, *args, mask=w.mask[:, :5].cuda())


@pytest.mark.parametrize("Lq", [20, 50])
@pytest.mark.parametrize("grow", [True, False])
def test_prefill_running_max_moves_across_tiles(grow, Lq, kernel):
    """Keys past position 300 scaled by 6 (exact in bf16): the logits of later tiles
    exceed the earlier maximum by far more than 2^8 (grow) or fall far below it; the
    tensor-core kernel rescales O in TMEM only in the first case."""
    w = case(12, D=128, Hq=8, Hkv=2, Lq=Lq, lens=(900, 700), causal=-1)
    P = w.k_cache.shape[1]
    for b, L in enumerate(w.seq_lens.tolist()):
        for t in range(300, L):
            page = int(w.page_table[b, t // P])
            if grow:
                w.k_cache[page, t % P] *= 6
            else:
                w.k_cache[page, t % P] /= 8
    check_close(run(w, kernel=kernel), oracle.paged_prefill(w), f"grow={grow}")


# ---------------------------------------------------------------- full size
@pytest.mark.parametrize("kernel_name", ["tcgen05", "mma_sync"])
def test_prefill_chunk_workload_full_size_sampled(kernel_name):
    """The bench's prefill workload at full size (16 sequences x 4096 keys, 128 causal
    queries, 32/8 heads, D = 128, shuffled 2048-page pool) in the bench's launch; three
    sequences are checked in full against the oracle, run on one-sequence slices of the
    same inputs (same pool, same page-table rows)."""
    w = workloads.prefill_llama8b_chunk()
    q = w.q.cuda()
    out = torch.full_like(q, float("nan"))
    apd.attn_paged_prefill(q, w.k_cache.cuda(), w.v_cache.cuda(), w.page_table.cuda(), w.seq_lens.cuda(), w.scale,
                           w.causal_offset, None, out, kernel=kernel_name)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    for b in (0, 7, 15):
        one = workloads.PrefillWorkload(name=f"{w.name}[{b}]", seed=w.seed, q=w.q[b:b + 1], k_cache=w.k_cache,
                                        v_cache=w.v_cache, page_table=w.page_table[b:b + 1],
                                        seq_lens=w.seq_lens[b:b + 1], scale=w.scale, causal_offset=w.causal_offset)
        check_close(out[b:b + 1], oracle.paged_prefill(one), f"{kernel_name} sequence {b}")
