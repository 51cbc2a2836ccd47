"""GPU parity of the tensor-core multi-query decode (plan mode 3: more than 16 q heads per kv
head at D = 128, decode_mq_tc_kernel with the heads padded to 32 or 64, above 64 cut into
blocks of q heads, merged in a cluster or by the fixed-split combine) against the fp64 CPU
oracle.

Per output element |gpu - ref| <= 1e-2 + 1e-2 |ref| (ref = fp64 oracle value), as for every
decode path.  Covered: automatic and fixed split counts (one split per unit, partial 128-token
tiles at the ends of splits, splits that get no token), lengths around the 32- and 128-token
tile edges with empty sequences, NaN-poisoned unused slots, pages of 64 tokens, HND storage,
the contiguous cache (bit-identical to the same tokens paged), scores with large outliers
and a large scale (the reference maximum moves mid-stream and O is rescaled), determinism,
CUDA-graph replay, the device-side contract flags, group sizes from 20 to 200 q heads per kv
head, and the full-size 32- and 80-heads-per-kv-head workloads in the launch configuration
the benchmark times.
"""
import numpy as np
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads
from gpu_util import DeviceProblem, check_close

pytestmark = pytest.mark.gpu


def small(seed, B, Hq, Hkv, lens, P=32, pool=None, **kw):
    return workloads.make(name="mq", seed=seed, batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128,
                          page_size=P, seq_lens=list(lens), pool_pages=pool, **kw)


def run_mode3(w, S, **kw):
    pl = apd.query_plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, S)
    assert pl.mode == 3
    dp = DeviceProblem(w)
    out = dp.run(S, **kw)
    return dp, out


@pytest.mark.parametrize("S", [0, 1, 2, 3, 4, 7, 16])
def test_ragged_with_empty_and_poison(S):
    w = small(2, 4, 64, 2, (1500, 0, 33, 777), pool=90, poison=True)
    dp, out = run_mode3(w, S)
    check_close(out, oracle.paged_decode(w), f"64/2 ragged S={S}")
    assert torch.all(out[1] == 0)
    assert apd.read_device_flags(dp.workspace) == 0


@pytest.mark.parametrize("S", [0, 3])
def test_lengths_around_tile_edges(S):
    # 1 token, 127/128/129 (one 128-token tile and its edges), 255, and a long one
    w = small(4, 6, 32, 1, (1, 127, 128, 129, 255, 4000), pool=200, poison=True)
    _, out = run_mode3(w, S)
    check_close(out, oracle.paged_decode(w), f"32/1 edges S={S}")


@pytest.mark.parametrize("S", [0, 2])
def test_larger_pages_and_more_kv_heads(S):
    w = small(5, 3, 128, 4, (700, 65, 1), P=64, pool=40, poison=True)
    _, out = run_mode3(w, S)
    check_close(out, oracle.paged_decode(w), f"128/4 P=64 S={S}")


def test_hnd_storage():
    w = small(6, 3, 64, 2, (900, 31, 200), pool=60, layout="HND", poison=True)
    _, out = run_mode3(w, 0)
    check_close(out, oracle.paged_decode(w), "64/2 HND")


@pytest.mark.parametrize("S", [0, 3])
def test_contig_matches_paged_bit_for_bit(S):
    wc = workloads.make_contig(name="mq_contig", seed=6, batch=3, num_q_heads=64, num_kv_heads=2, head_dim=128,
                               seq_lens=[300, 1, 90], lmax=333)
    wp = workloads.paged_from_contig(wc, page_size=32, seed=2)
    a = DeviceProblem(wc).run(S).clone()
    b = DeviceProblem(wp).run(S).clone()
    assert torch.equal(a, b)
    check_close(a, oracle.paged_decode(wc), f"contig S={S}")


@pytest.mark.parametrize("S", [0, 1, 5])
def test_score_outliers_move_the_reference(S):
    """Keys with 30x outliers, and a unit scale (scores of tens), so that some head's
    maximum grows by more than 2^8 after the first tile: O^T and the running sums are
    rescaled mid-stream."""
    w = small(7, 3, 64, 2, (3000, 2500, 40), pool=250, k_outlier_frac=0.02, k_outlier_mult=30.0)
    _, out = run_mode3(w, S)
    check_close(out, oracle.paged_decode(w), f"outliers S={S}")
    w = small(8, 2, 64, 2, (4000, 1000), pool=200, scale=1.0, k_outlier_frac=0.01)
    _, out = run_mode3(w, S)
    check_close(out, oracle.paged_decode(w), f"unit scale S={S}")


@pytest.mark.parametrize("S", [0, 4])
def test_deterministic(S):
    w = small(9, 4, 64, 2, (2000, 100, 3333, 7), pool=200)
    dp = DeviceProblem(w)
    a = dp.run(S).clone()
    b = dp.run(S).clone()
    assert torch.equal(a, b)


def test_cuda_graph_capture_and_replay():
    w1 = small(10, 4, 64, 2, (1000, 2000, 5, 0), pool=100)
    w2 = small(11, 4, 64, 2, (1000, 2000, 5, 0), pool=100)
    dp = DeviceProblem(w1)
    ws = apd.alloc_workspace(4, 64, 2, 128, 0)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        call = apd.DecodeCall(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w1.scale, 0, ws)
        call(st)  # warm-up outside the capture
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            call(st)
    g.replay()
    torch.cuda.synchronize()
    check_close(dp.out, oracle.paged_decode(w1), "graph replay 1")
    # new values in the same buffers, replayed
    dp.q.copy_(w2.q.to("cuda"))
    dp.k.copy_(w2.k_cache.to("cuda"))
    dp.v.copy_(w2.v_cache.to("cuda"))
    dp.page_table.copy_(w2.page_table.to("cuda"))
    g.replay()
    torch.cuda.synchronize()
    check_close(dp.out, oracle.paged_decode(w2), "graph replay 2")


def test_contract_flags():
    w = small(12, 3, 64, 2, (300, 64, 100), pool=20, max_pages_per_seq=10)
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    dp.page_table[1, 0] = w.num_pages + 3  # out of range: read as zeros, flagged
    dp.seq_lens[2] = -7                     # treated as 0, flagged
    ws = apd.alloc_workspace(3, 64, 2, 128, 0)
    apd.workspace_init(ws)
    apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws)
    flags = apd.read_device_flags(ws)
    assert flags & apd.FLAG_PAGE_OUT_OF_RANGE and flags & apd.FLAG_SEQ_LEN_NEGATIVE
    out = dp.out.to(torch.float64).cpu().numpy()
    assert np.isfinite(out).all()
    assert np.all(out[2] == 0)
    check_close(dp.out[[0]], ref[[0]], "untouched sequence")


@pytest.mark.parametrize("g", [20, 48, 64])
@pytest.mark.parametrize("S", [0, 1, 3, 16])
def test_other_group_sizes(g, S):
    """Group sizes padded to the kernel's 32 or 64 heads (20 -> 32; 48, 64 -> 64: the softmax
    in two passes of 32 heads): ragged lengths with an empty sequence, poisoned slots, and
    score outliers that move the reference maximum of some heads."""
    w = small(13, 4, 2 * g, 2, (1900, 0, 77, 640), pool=120, poison=True, k_outlier_frac=0.02,
              k_outlier_mult=20.0)
    dp, out = run_mode3(w, S)
    check_close(out, oracle.paged_decode(w), f"g={g} S={S}")
    assert torch.all(out[1] == 0)
    assert apd.read_device_flags(dp.workspace) == 0


def test_gqa32_full_size():
    w = workloads.gqa32()
    pl = apd.query_plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, 0)
    assert pl.mode == 3
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    check_close(dp.run(0), ref, "gqa32 auto")
    check_close(dp.run(16), ref, "gqa32 S=16")
    assert apd.read_device_flags(dp.workspace) == 0


@pytest.mark.parametrize("g,Hkv", [(65, 2), (80, 2), (128, 1), (200, 1)])
@pytest.mark.parametrize("S", [0, 1, 3, 16])
def test_q_head_blocks(g, Hkv, S):
    """More than 64 q heads per kv head: ceil(g / 64) blocks of q heads, one CTA per block
    and split (65 -> 48 + 17, 80 -> 48 + 32, 128 -> 64 + 64, 200 -> 64 + 64 + 64 + 8), the
    blocks after the first starting inside the 16-row slot layout of the partials.  Ragged
    lengths with an empty sequence, poisoned slots, score outliers."""
    w = small(14, 4, g * Hkv, Hkv, (1900, 0, 77, 640), pool=120, poison=True, k_outlier_frac=0.02,
              k_outlier_mult=20.0)
    pl = apd.query_plan(4, g * Hkv, Hkv, 128, S)
    nb = -(-g // 64)
    assert pl.q_head_blocks == nb and pl.grid_ctas % (4 * Hkv * nb) == 0
    dp, out = run_mode3(w, S)
    check_close(out, oracle.paged_decode(w), f"g={g} S={S}")
    assert torch.all(out[1] == 0)
    assert apd.read_device_flags(dp.workspace) == 0


def test_q_head_blocks_contract_flags():
    """Page-table and length violations seen by the CTA of every block of q heads are
    flagged once in the shared flag word, and the other sequences stay exact."""
    w = small(15, 3, 160, 2, (300, 64, 100), pool=20, max_pages_per_seq=10)
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    dp.page_table[1, 0] = w.num_pages + 3
    dp.seq_lens[2] = -7
    ws = apd.alloc_workspace(3, 160, 2, 128, 0)
    apd.workspace_init(ws)
    apd.attn_paged_decode(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, 0, ws)
    flags = apd.read_device_flags(ws)
    assert flags & apd.FLAG_PAGE_OUT_OF_RANGE and flags & apd.FLAG_SEQ_LEN_NEGATIVE
    out = dp.out.to(torch.float64).cpu().numpy()
    assert np.isfinite(out).all() and np.all(out[2] == 0)
    check_close(dp.out[[0]], ref[[0]], "untouched sequence")


def test_gqa80_full_size():
    w = workloads.gqa80()
    pl = apd.query_plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, 0)
    assert pl.mode == 3 and pl.q_head_blocks == 2 and pl.q_heads_per_block == 48
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    check_close(dp.run(0), ref, "gqa80 auto")
    check_close(dp.run(16), ref, "gqa80 S=16")
    assert apd.read_device_flags(dp.workspace) == 0
