"""Failure detection on the GPU without a fault: the bounded waits that every kernel uses
on its mbarriers give up, report a status the host reads, and leave the context usable.

The self-test waits on mbarriers that nothing completes (no copy, MMA or fault): the
first wait has a 1 ms limit and must give up and raise the CTA's abort flag; the second
has the kernels' full 2 s limit and must give up early because of that flag."""
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads
from gpu_util import DeviceProblem, check_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_it():
    first, second, second_us, flags = apd.selftest_bounded_wait(1_000_000)
    assert first == 1 and flags & apd.FLAG_WAIT_TIMEOUT
    assert second == 1
    assert 500 <= second_us <= 100_000, second_us  # ended through the abort flag, far below 2 s


def test_context_is_usable_after_a_wait_gave_up():
    apd.selftest_bounded_wait(200_000)
    w = workloads.make(name="after", seed=61, batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128,
                       seq_lens=[100, 7, 64], page_size=32)
    dp = DeviceProblem(w)
    check_close(dp.run(0), oracle.paged_decode(w), "decode after the self-test")


def test_shared_ring_leader_stops_when_a_release_never_comes():
    """The shared K/V ring's error path (80 q heads per kv head at D = 64, auto splits): the
    self-test runs the real decode with followers that never release a stage and a 1 ms
    limit per wait.  Each ring's leader must give up at its first refill, stop issuing and
    return, and its followers must stop through the CTA's abort word, so the call ends
    within a few limits (a leader that kept refilling would wait out one limit per tile:
    over 100 ms here) with APD_FLAG_WAIT_TIMEOUT set.  A normal call afterwards is correct."""
    w = workloads.make(name="ring_release", seed=83, batch=4, num_q_heads=160, num_kv_heads=2, head_dim=64,
                       seq_lens=[16384, 16000, 12000, 16384], page_size=32)
    dp = DeviceProblem(w)
    default = apd.workspace_size(4, 160, 2, 64, 0)
    ws = torch.zeros(default // 16 // 256 * 256, dtype=torch.uint8, device="cuda")  # long runs per warp
    plan = apd.query_plan(4, 160, 2, 64, 0, workspace_bytes=ws.numel())
    assert plan.shared_kv_ring == 1 and plan.mode == 0
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    apd.selftest_shared_ring_release(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, ws, 1_000_000)
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    assert apd.read_device_flags(ws) & apd.FLAG_WAIT_TIMEOUT
    assert ms < 30.0, f"the self-test call took {ms:.1f} ms"
    check_close(dp.run(0, workspace=ws), oracle.paged_decode(w), "decode after the release self-test")
    assert apd.read_device_flags(ws) == 0


def test_release_selftest_needs_the_shared_ring():
    w = workloads.make(name="no_ring", seed=84, batch=2, num_q_heads=32, num_kv_heads=8, head_dim=128,
                       seq_lens=[64, 96], page_size=32)
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(2, 32, 8, 128, 0)
    with pytest.raises(apd.APDError):
        apd.selftest_shared_ring_release(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, ws)


@pytest.mark.parametrize("B,S,Hq", [(16, 0, 64), (4, 0, 64), (16, 16, 64), (8, 0, 160)])
def test_tensor_core_kernel_stops_when_a_hand_over_never_comes(B, S, Hq):
    """The tensor-core multi-query kernel's error path (32 q heads per kv head at D = 128),
    with the splits merged in a cluster (B = 16, auto: 4 splits) or by the combine (B = 4,
    auto: 16 splits; B = 16 with 16 fixed splits); and 80 q heads per kv head in two blocks
    of q heads (B = 8, auto: 4 splits, in a cluster where the device holds 32 of them).  The
    self-test runs the real decode with softmax warps that never hand over the weights of
    their second tile and a 1 ms limit per wait: the MMA issuer and the softmax warps must give up, leave their loops together,
    wait for their copies and MMAs in flight, free TMEM and meet at the cluster barrier, so
    the call ends within a few limits with APD_FLAG_WAIT_TIMEOUT set.  A normal call
    afterwards is correct."""
    w = workloads.make(name="mq_stall", seed=85, batch=B, num_q_heads=Hq, num_kv_heads=2, head_dim=128,
                       seq_lens=[16384] * B, page_size=32)
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(B, Hq, 2, 128, S)
    plan = apd.query_plan(B, Hq, 2, 128, S)
    assert plan.mode == 3 and plan.q_head_blocks == (2 if Hq == 160 else 1)
    if Hq == 64:
        assert (plan.cluster_size > 0) == (B == 16 and S == 0)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    apd.selftest_mq_tc_stall(dp.q, dp.k, dp.v, dp.page_table, dp.seq_lens, dp.out, w.scale, S, ws, 1_000_000)
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    assert apd.read_device_flags(ws) & apd.FLAG_WAIT_TIMEOUT
    assert ms < 30.0, f"the self-test call took {ms:.1f} ms"
    check_close(dp.run(S, workspace=ws), oracle.paged_decode(w), "decode after the stall self-test")
    assert apd.read_device_flags(ws) == 0
