"""GPU parity of the decode projection GEMV (apd_gemv_bf16) against the fp64 oracle.

Per element: |gpu - ref| <= 2^-8 |ref| + 2^-13 sum_k |x w|, i.e. the bf16 rounding
of the output (at most one ulp allowed) plus fp32 accumulation error scaled by the
magnitude of the terms.  Shapes cover every M in 1..8, N and K tails, strided
operands, tiny and very wide layers, and the AstrAI-1B projection shapes at full
size."""
import numpy as np
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads

pytestmark = pytest.mark.gpu


def check(y, x, w, what=""):
    ref, absref = oracle.gemv(x, w)
    got = y.to(torch.float64).cpu().numpy()
    assert np.isfinite(got).all(), what
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -13 * absref
    assert (err <= bound).all(), f"{what}: max err {err.max():.3e}, worst ratio {(err / bound).max():.2f}"


@pytest.mark.parametrize("M", range(1, 9))
@pytest.mark.parametrize("N,K", [(64, 256), (37, 1000), (1, 8), (300, 4104), (16, 264), (50, 1040), (3000, 1000),
                                 (9470, 2048)])
def test_gemv_shapes(M, N, K):
    c = workloads.gemv_case(M, N, K, seed=M * 7 + N)
    y = apd.gemv(c.x.cuda(), c.w.cuda())
    check(y, c.x, c.w, f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(1, 64, 520), (8, 1000, 6920), (3, 2360, 1040), (2, 16, 512), (5, 33, 8200),
                                   (7, 1536, 6912)])
def test_gemv_one_cta_per_mtile(M, N, K):
    """Short weight streams with fewer 16-row tiles than SMs: one CTA per tile, whose warps
    split its k-tiles (3 k-tiles on 3 warps, 28 with a K tail, 5, 2, 33 on 4 warps) and add
    their parts in shared memory; N tails (1000, 33) and the full 148 tiles (2360)."""
    plan = apd.gemv_query_plan(M, N, K)
    assert plan["cta_per_mtile"] == 1 and plan["sum_ctas"] == 0
    c = workloads.gemv_case(M, N, K, seed=N + K)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(apd.gemv_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    apd.gemv(c.x.cuda(), c.w.cuda(), y, ws)
    check(y, c.x, c.w, f"cta per m-tile M={M} N={N} K={K}")
    assert apd.read_device_flags(ws) == 0


def test_gemv_strided_operands():
    c = workloads.gemv_case(5, 200, 512, seed=3)
    xb = torch.zeros(5, 640, dtype=torch.bfloat16, device="cuda")
    xb[:, 64:576] = c.x.cuda()
    wb = torch.zeros(200, 528, dtype=torch.bfloat16, device="cuda")
    wb[:, 8:520] = c.w.cuda()
    yt = torch.full((200, 5), float("nan"), dtype=torch.bfloat16, device="cuda")  # y as a transposed view
    apd.gemv(xb[:, 64:576], wb[:, 8:520], yt.t())
    check(yt.t(), c.x, c.w, "strided")


@pytest.mark.parametrize("layer", list(workloads.GEMV_SHAPES))
@pytest.mark.parametrize("M", [1, 3, 8])
def test_gemv_projection_shapes(layer, M):
    c = workloads.gemv_named(layer, M)
    check(apd.gemv(c.x.cuda(), c.w.cuda()), c.x, c.w, f"{layer} M={M}")


@pytest.mark.parametrize("M,N,K,pad", [(5, 22000, 1544, 8), (8, 21000, 1600, 0), (1, 22000, 1544, 0)])
def test_gemv_x_staged_once_per_cta(M, N, K, pad):
    """Weights of 64 MB and more take the path that copies x into shared memory once per
    CTA: an odd number of 16-byte chunks per row with a partial last 256-column tile
    (K = 1544), an even number that needs the padded row pitch (K = 1600), a strided x."""
    c = workloads.gemv_case(M, N, K, seed=21)
    xb = torch.zeros(M, K + pad, dtype=torch.bfloat16, device="cuda")
    xb[:, :K] = c.x.cuda()
    y = apd.gemv(xb[:, :K], c.w.cuda())
    check(y, c.x, c.w, f"staged x M={M} N={N} K={K} pad={pad}")


def test_gemv_graph_capture_and_repeat():
    c = workloads.gemv_case(4, 1000, 2048, seed=9)
    x, w = c.x.cuda(), c.w.cuda()
    ws = torch.zeros(apd.gemv_workspace_size(4, 1000, 2048), dtype=torch.uint8, device="cuda")
    y = torch.empty(4, 1000, dtype=torch.bfloat16, device="cuda")
    apd.gemv(x, w, y, ws)
    first = y.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            apd.gemv(x, w, y, ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, first)  # deterministic


def test_gemv_rejects_bad_arguments():
    x = torch.zeros(9, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Exception):
        apd.gemv(x, w)  # M > 8
    with pytest.raises(apd.APDError):
        apd.gemv(torch.zeros(2, 60, dtype=torch.bfloat16, device="cuda"),
                 torch.zeros(16, 60, dtype=torch.bfloat16, device="cuda"),
                 workspace=torch.zeros(1 << 20, dtype=torch.uint8, device="cuda"))  # K % 8 != 0
