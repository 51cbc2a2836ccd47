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
