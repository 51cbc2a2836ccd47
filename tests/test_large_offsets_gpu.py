"""GPU parity when the data a call reads lies past element 2^31 of its cache.

Every K/V access goes through TMA tensor maps (64-bit byte strides, 32-bit
coordinates), and q / out / mask through 64-bit strides; these cases pin that on
caches of 4.5-7 GB each, for the split, unit and tensor-core decode kernels and both
prefill kernels.  Only the pages (or rows) a call references are filled
with the workload's seeded values, placed at the far end of a large allocation whose
other contents are never written and must never be read; the oracle sees the
compact workload.  Per element |gpu - ref| <= 1e-2 + 1e-2 |ref|, as everywhere."""
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads
from gpu_util import DeviceProblem, check_close

pytestmark = pytest.mark.gpu

TWO31 = 2 ** 31


@pytest.fixture(autouse=True)
def _release_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def far_pool(cache: torch.Tensor, pages_needed: int):
    """A [NP, ...] device pool whose last `pages_needed` pages hold `cache` and start
    past element 2^31; returns (pool, index of its first filled page)."""
    per_page = cache[0].numel()
    base = TWO31 // per_page + 1
    pool = torch.empty((base + pages_needed,) + tuple(cache.shape[1:]), dtype=cache.dtype, device="cuda")
    pool[base:] = cache
    assert base * per_page > TWO31
    return pool, base


@pytest.mark.parametrize("S", [0, 1, 4])
def test_paged_decode_pages_past_2_31_elements(S):
    w = workloads.make(name="far", seed=61, batch=3, num_q_heads=16, num_kv_heads=2, head_dim=128, page_size=32,
                       seq_lens=[1000, 700, 33], pool_pages=64)
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    k, base = far_pool(dp.k, dp.k.shape[0])
    v, _ = far_pool(dp.v, dp.v.shape[0])
    pt = dp.page_table + base
    ws = apd.alloc_workspace(3, 16, 2, 128, S)
    apd.attn_paged_decode(dp.q, k, v, pt, dp.seq_lens, dp.out, w.scale, S, ws)
    check_close(dp.out, ref, f"pages past 2^31 S={S}")
    assert apd.read_device_flags(ws) == 0


@pytest.mark.parametrize("Hq,S", [(64, 0), (64, 3), (64, 16), (96, 0)])
def test_tensor_core_decode_pages_past_2_31_elements(Hq, S):
    """The tensor-core multi-query kernel (32 and 48 q heads per kv head at D = 128), with
    its splits merged in a cluster (auto, 3) or by the combine (16)."""
    w = workloads.make(name="far", seed=64, batch=3, num_q_heads=Hq, num_kv_heads=2, head_dim=128, page_size=32,
                       seq_lens=[1000, 700, 33], pool_pages=64)
    assert apd.query_plan(3, Hq, 2, 128, S).mode == 3
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    k, base = far_pool(dp.k, dp.k.shape[0])
    v, _ = far_pool(dp.v, dp.v.shape[0])
    pt = dp.page_table + base
    ws = apd.alloc_workspace(3, Hq, 2, 128, S)
    apd.attn_paged_decode(dp.q, k, v, pt, dp.seq_lens, dp.out, w.scale, S, ws)
    check_close(dp.out, ref, f"tensor-core pages past 2^31 {Hq}/2 S={S}")
    assert apd.read_device_flags(ws) == 0


def test_contig_decode_rows_past_2_31_elements():
    lens = [300, 517, 1000]
    w = workloads.make_contig(name="far", seed=62, batch=3, num_q_heads=16, num_kv_heads=2, head_dim=128,
                              seq_lens=lens, lmax=1024, layout="blhd")
    ref = oracle.paged_decode(w)
    dp = DeviceProblem(w)
    # [B, Lmax, Hkv, D] with Lmax large enough that sequence 2 starts past element 2^31
    lmax = TWO31 // (2 * 2 * 128) + 1024
    k = torch.empty((3, lmax, 2, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    k[:, :1024] = dp.k
    v[:, :1024] = dp.v
    assert 2 * lmax * 2 * 128 > TWO31
    ws = apd.alloc_workspace(3, 16, 2, 128, 0)
    apd.attn_contig_decode(dp.q, k, v, dp.seq_lens, dp.out, w.scale, 0, ws)
    check_close(dp.out, ref, "contig rows past 2^31")


@pytest.mark.parametrize("kernel", ["mma_sync", "tcgen05"])
@pytest.mark.parametrize("Lq", [5, 45])
def test_prefill_pages_past_2_31_elements(kernel, Lq):
    """Lq = 45 with 8 query heads per kv head gives 360 rows: the two-tile tensor-core kernel."""
    w = workloads.make_prefill(name="far", seed=63, batch=2, q_len=Lq, num_q_heads=16, num_kv_heads=2, head_dim=128,
                               seq_lens=[600, 260], page_size=32, causal_offset=555, max_pages_per_seq=19)
    ref = oracle.paged_prefill(w)
    kc, vc = w.k_cache.contiguous().cuda(), w.v_cache.contiguous().cuda()
    k, base = far_pool(kc, kc.shape[0])
    v, _ = far_pool(vc, vc.shape[0])
    q = w.q.cuda()
    out = torch.full_like(q, float("nan"))
    apd.attn_paged_prefill(q, k, v, w.page_table.cuda() + base, w.seq_lens.cuda(), w.scale, w.causal_offset, None,
                           out, kernel=kernel)
    torch.cuda.synchronize()
    check_close(out, ref, f"prefill pages past 2^31 {kernel} Lq={Lq}")
