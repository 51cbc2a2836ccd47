"""Pins of the fp64 multi-query (prefill) oracle against things other than itself.

* brute force: K/V gathered by a plain loop and a visibility matrix built element by
  element from the causal offset, the lengths and the mask, given to torch's fp64
  scaled_dot_product_attention (a library routine);
* special cases: one query with no causal offset and no mask is single-token decode
  (the separately pinned decode oracle); causal offset 0 makes query 0 see key 0
  only (its output is V[0] exactly); an all-ones mask changes nothing; a query that
  sees no key gives zeros.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads


def brute(w):
    B, Lq, Hq, D = w.q.shape
    Hkv, P = w.k_cache.shape[2], w.k_cache.shape[1]
    g = Hq // Hkv
    out = np.zeros((B, Lq, Hq, D))
    seen = np.zeros((B, Lq), dtype=bool)
    kc, vc = w.k_cache.to(torch.float64), w.v_cache.to(torch.float64)
    for b in range(B):
        L = int(w.seq_lens[b])
        if L == 0:
            continue
        K = torch.empty(Hkv, L, D, dtype=torch.float64)
        V = torch.empty(Hkv, L, D, dtype=torch.float64)
        for t in range(L):
            page = int(w.page_table[b, t // P])
            K[:, t], V[:, t] = kc[page, t % P], vc[page, t % P]
        vis = torch.zeros(Lq, L, dtype=torch.bool)
        for i in range(Lq):
            for t in range(L):
                ok = w.causal_offset < 0 or t <= w.causal_offset + i
                if w.mask is not None:
                    ok = ok and bool(w.mask[b, t] if w.mask.dim() == 2 else w.mask[b, i, t])
                vis[i, t] = ok
        rows = vis.any(1)
        seen[b] = rows.numpy()
        if not rows.any():
            continue
        q = w.q[b].to(torch.float64).permute(1, 0, 2)  # [Hq, Lq, D]
        o = F.scaled_dot_product_attention(q[:, rows], K.repeat_interleave(g, 0), V.repeat_interleave(g, 0),
                                           attn_mask=vis[rows], scale=w.scale)
        out[b, rows.numpy()] = o.permute(1, 0, 2).numpy()
    return out, seen


CASES = [
    dict(batch=2, q_len=5, num_q_heads=4, num_kv_heads=2, head_dim=16, seq_lens=[40, 9], page_size=8,
         causal_offset=35, mask=None),
    dict(batch=2, q_len=6, num_q_heads=6, num_kv_heads=3, head_dim=32, seq_lens=[23, 30], page_size=4,
         causal_offset=-1, mask="2d"),
    dict(batch=3, q_len=4, num_q_heads=8, num_kv_heads=2, head_dim=16, seq_lens=[17, 1, 12], page_size=4,
         causal_offset=10, mask="3d", mask_keep=0.6),
    dict(batch=1, q_len=7, num_q_heads=2, num_kv_heads=1, head_dim=64, seq_lens=[33], page_size=32,
         causal_offset=0, mask=None),
]


@pytest.mark.parametrize("cfg", CASES)
def test_brute_force(cfg):
    w = workloads.make_prefill(name="pin", seed=17, **cfg)
    ref, seen = brute(w)
    got = oracle.paged_prefill(w)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    assert np.all(got[~seen] == 0)  # a query that sees no key gives zeros


def test_single_query_is_decode():
    w = workloads.make_prefill(name="d", seed=5, batch=3, q_len=1, num_q_heads=8, num_kv_heads=2, head_dim=32,
                               seq_lens=[5, 40, 17], page_size=8)
    dec = workloads.Workload(name="d", seed=5, q=w.q[:, 0], k_cache=w.k_cache, v_cache=w.v_cache,
                             page_table=w.page_table, seq_lens=w.seq_lens, scale=w.scale)
    assert np.array_equal(oracle.paged_prefill(w)[:, 0], oracle.paged_decode(dec))


def test_causal_offset_zero_first_query_sees_key_zero():
    w = workloads.make_prefill(name="c", seed=6, batch=2, q_len=3, num_q_heads=4, num_kv_heads=1, head_dim=16,
                               seq_lens=[10, 3], page_size=4, causal_offset=0)
    got = oracle.paged_prefill(w)
    for b in range(2):
        page = int(w.page_table[b, 0])
        v0 = w.v_cache[page, 0, 0].to(torch.float64).numpy()
        for h in range(4):
            assert np.array_equal(got[b, 0, h], v0)


def test_all_ones_mask_changes_nothing():
    w = workloads.make_prefill(name="m", seed=7, batch=2, q_len=4, num_q_heads=4, num_kv_heads=2, head_dim=16,
                               seq_lens=[25, 14], page_size=8, causal_offset=20, mask="3d")
    w.mask.fill_(1)
    a = oracle.paged_prefill(w)
    w.mask = None
    assert np.array_equal(a, oracle.paged_prefill(w))


def test_masked_out_row_is_zero():
    w = workloads.make_prefill(name="z", seed=8, batch=1, q_len=3, num_q_heads=2, num_kv_heads=1, head_dim=16,
                               seq_lens=[12], page_size=4, mask="3d")
    w.mask[0, 1] = 0
    got = oracle.paged_prefill(w)
    assert np.all(got[0, 1] == 0) and np.any(got[0, 0] != 0)
