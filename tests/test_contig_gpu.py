"""GPU parity of the contiguous-KV call (ContigKV policy, "blhd" and "bhld" layouts)
against the fp64 oracle, and bit-for-bit agreement with the paged call on the same
tokens (the pages' paged-versus-contiguous test)."""
import numpy as np
import pytest
import torch

import decode_attention_paged_split_b200 as apd
import oracle
import workloads
from gpu_util import DeviceProblem, check_close

pytestmark = pytest.mark.gpu


def contig(seed, D, lens, lmax, layout="blhd", Hq=16, Hkv=4, **kw):
    return workloads.make_contig(name="contig", seed=seed, batch=len(lens), num_q_heads=Hq, num_kv_heads=Hkv,
                                 head_dim=D, seq_lens=list(lens), lmax=lmax, layout=layout, **kw)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("layout", ["blhd", "bhld"])
@pytest.mark.parametrize("S", [0, 1, 4])
def test_contig_matches_oracle(D, layout, S):
    # Lmax = 1000 is not a multiple of 32: the last tile's rows past Lmax are outside the tensor
    w = contig(5, D, (0, 1, 31, 32, 33, 517, 1000), 1000, layout)
    ref = oracle.paged_decode(w)
    out = DeviceProblem(w).run(S)
    check_close(out, ref, f"contig D={D} {layout} S={S}")
    assert torch.all(out[0] == 0)


@pytest.mark.parametrize("S", [0, 1, 3, 148])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (40, 2)])
def test_paged_and_contig_agree_bit_for_bit(S, Hq, Hkv):
    w = contig(6, 128, (700, 64, 1500, 1, 0, 2048), 2048, "blhd", Hq=Hq, Hkv=Hkv)
    wp = workloads.paged_from_contig(w, page_size=32, seed=2)
    a = DeviceProblem(w).run(S).clone()
    b = DeviceProblem(wp).run(S).clone()
    assert torch.equal(a, b)
    check_close(a, oracle.paged_decode(w), f"contig vs oracle S={S}")


def test_contig_cuda_graph():
    w = contig(7, 128, (300, 77, 1024), 1024, "bhld", Hq=32, Hkv=8)
    dp = DeviceProblem(w)
    ws = apd.alloc_workspace(3, 32, 8, 128, 0)
    call = apd.DecodeCall(dp.q, dp.k, dp.v, None, dp.seq_lens, dp.out, w.scale, 0, ws)
    call()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            call(s)
    torch.cuda.current_stream().wait_stream(s)
    dp.out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    check_close(dp.out, oracle.paged_decode(w), "contig graph replay")


def test_contig_llama8b_full_size():
    w = workloads.llama8b_contig()
    check_close(DeviceProblem(w).run(0), oracle.paged_decode(w), "llama8b contig")


def test_contig_lengths_past_lmax_are_clamped():
    w = contig(8, 64, (40, 64), 64, "blhd", Hq=4, Hkv=1, poison=False)
    dp = DeviceProblem(w)
    dp.seq_lens[1] = 500
    ws = apd.alloc_workspace(2, 4, 1, 64, 0)
    apd.workspace_init(ws)
    apd.attn_contig_decode(dp.q, dp.k, dp.v, dp.seq_lens, dp.out, w.scale, 0, ws)
    assert apd.read_device_flags(ws) & apd.FLAG_SEQ_LEN_CLAMPED
    check_close(dp.out, oracle.paged_decode(w), "clamped to Lmax")
