"""apd_attn_paged_decode_noalloc: the entry point for callers that cannot allocate
device memory (a plugin handed only its tensors by a framework that owns every
allocation, code under a fixed memory budget, or a latency path where cudaMalloc's
implicit synchronisation is not acceptable).  It takes no workspace and uses the
library's built-in static device scratch instead.

The GPU test calls it through the C ABI (ctypes, no binding helper) twice in a row,
so the second call runs on scratch the first one left behind. Each time it
compares the output with the workspace entry point's and with the fp64 oracle,
within the tolerance of the parity tests.  This file is named so that pytest
collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads
from gpu_util import check_close

SCRATCH_LIMIT = 13  # APD_ERR_SCRATCH_LIMIT
ATOL = RTOL = 1e-2  # the parity tests' per-element bound


def _descs(*ts):
    return [apd._desc(t) for t in ts]


def _call_noalloc(q, k, v, pt, sl, out, scale, splits, stream=None):
    d = _descs(q, k, v, pt, sl, out)
    return apd.lib().apd_attn_paged_decode_noalloc(*[ctypes.byref(x) for x in d], ctypes.c_float(scale),
                                                   int(splits), stream)


def test_oversized_problem_is_rejected_before_any_launch():
    """Host-side size check: 512 units x 148 splits of fp32 partials cannot fit in 8 MiB."""
    B, Hq, Hkv, D = 64, 32, 8, 256
    assert apd.workspace_size(B, Hq, Hkv, D, 148) > apd.NOALLOC_SCRATCH_BYTES
    fake = 1 << 32
    q = apd._Tensor(); k = apd._Tensor(); v = apd._Tensor(); pt = apd._Tensor(); sl = apd._Tensor(); o = apd._Tensor()
    for t, shape, dt in ((q, [B, Hq, D], 1), (o, [B, Hq, D], 1), (k, [64, 32, Hkv, D], 1), (v, [64, 32, Hkv, D], 1),
                         (pt, [B, 8], 2), (sl, [B], 2)):
        t.data, t.dtype, t.ndim = fake, dt, len(shape)
        acc = 1
        for i in reversed(range(len(shape))):
            t.shape[i] = shape[i]
            t.stride[i] = acc
            acc *= shape[i]
    rc = apd.lib().apd_attn_paged_decode_noalloc(*[ctypes.byref(x) for x in (q, k, v, pt, sl, o)],
                                                 ctypes.c_float(0.1), 148, None)
    assert rc == SCRATCH_LIMIT
    assert "APD_NOALLOC_SCRATCH_BYTES" in apd.status_string(SCRATCH_LIMIT)


CASES = [
    ("sweep_d128_g4_auto", lambda: workloads.sweep_case(128, 32, 8, 0), 0),
    ("sweep_d64_g1_split4", lambda: workloads.sweep_case(64, 8, 8, 4), 4),
    ("ragged_g20_d256_split3", lambda: workloads.make(name="g20", seed=5, batch=3, num_q_heads=40, num_kv_heads=2,
                                                      head_dim=256, page_size=32, seq_lens=[0, 700, 33],
                                                      pool_pages=40, poison=True, max_pages_per_seq=24), 3),
    ("llama8b_auto", lambda: workloads.llama8b(), 0),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,make,splits", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry_twice(name, make, splits):
    w = make()
    dev = "cuda"
    q, k, v = w.q.to(dev), w.k_cache.contiguous().to(dev), w.v_cache.contiguous().to(dev)
    pt, sl = w.page_table.to(dev), w.seq_lens.to(dev)
    ref_out = torch.full_like(q, float("nan"))
    ws = apd.alloc_workspace(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, splits)
    apd.attn_paged_decode(q, k, v, pt, sl, ref_out, w.scale, splits, ws)
    ref = ref_out.to(torch.float64).cpu().numpy()
    assert np.isfinite(ref).all()
    oref = oracle.paged_decode(w)
    stream = torch.cuda.current_stream().cuda_stream or None
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        rc = _call_noalloc(q, k, v, pt, sl, out, w.scale, splits, stream)
        assert rc == 0, apd.status_string(rc)
        torch.cuda.synchronize()
        got = out.to(torch.float64).cpu().numpy()
        assert np.isfinite(got).all(), f"{name} call {call}: non-finite output"
        err = np.abs(got - ref)
        assert (err <= ATOL + RTOL * np.abs(ref)).all(), f"{name} call {call}: max err {err.max():.3e}"
        check_close(out, oref, f"{name} call {call} against the oracle")
