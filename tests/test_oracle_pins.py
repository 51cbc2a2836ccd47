"""Pins for the fp64 CPU oracle: it is checked against things other than itself.

* brute force: contiguous K/V gathered by a plain Python loop, GQA expanded with
  repeat_interleave, then torch's fp64 scaled_dot_product_attention (a library
  routine with none of the oracle's code);
* closed forms: L = 1 gives V[0]; constant K or q = 0 gives the mean of V; a
  huge scale with a unique maximum logit gives V[argmax]; L = 0 gives 0;
* a hand-derived golden example (tests/golden/hand_example_gqa.json);
* invariants: a permuted physical page placement gives a bit-identical result,
  split-and-combine at any split count or partition equals no split, GQA equals
  MHA with K/V repeated per query head, NaN in slots that must not be read
  changes nothing;
* bf16 rounding: hand examples (ties to even, overflow) and agreement with
  torch's float32 -> bf16 conversion on float32-representable values.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_force(w) -> np.ndarray:
    """Gather pages into contiguous K/V with a plain loop, then library SDPA in fp64."""
    B, Hq, D = w.q.shape
    Hkv = w.k_cache.shape[2]
    P = w.k_cache.shape[1]
    g = Hq // Hkv
    out = np.zeros((B, Hq, D))
    kc = w.k_cache.to(torch.float64)
    vc = w.v_cache.to(torch.float64)
    for b in range(B):
        L = int(w.seq_lens[b])
        if L == 0:
            continue
        K = torch.empty(Hkv, L, D, dtype=torch.float64)
        V = torch.empty(Hkv, L, D, dtype=torch.float64)
        for t in range(L):
            page = int(w.page_table[b, t // P])
            K[:, t] = kc[page, t % P]
            V[:, t] = vc[page, t % P]
        K = K.repeat_interleave(g, dim=0)
        V = V.repeat_interleave(g, dim=0)
        q = w.q[b].to(torch.float64)[:, None, :]
        o = F.scaled_dot_product_attention(q, K, V, scale=w.scale)
        out[b] = o[:, 0, :].numpy()
    return out


def small(seed, B=3, Hq=4, Hkv=2, D=32, P=4, lens=(5, 1, 13), pool=None, **kw):
    return workloads.make(name="pin", seed=seed, batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                          page_size=P, seq_lens=list(lens), pool_pages=pool, **kw)


@pytest.mark.parametrize("cfg", [
    dict(B=3, Hq=4, Hkv=2, D=32, P=4, lens=(5, 1, 13)),
    dict(B=2, Hq=8, Hkv=8, D=16, P=8, lens=(17, 40), pool=20),
    dict(B=1, Hq=6, Hkv=1, D=64, P=32, lens=(97,), pool=9),
    dict(B=4, Hq=4, Hkv=4, D=8, P=2, lens=(2, 3, 7, 1)),
    dict(B=2, Hq=16, Hkv=2, D=32, P=16, lens=(33, 64), layout="HND"),
])
def test_brute_force(cfg):
    w = small(11, **cfg)
    ref = brute_force(w)
    got = oracle.paged_decode(w)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_brute_force_workload_tiny():
    w = workloads.tiny()
    np.testing.assert_allclose(oracle.paged_decode(w), brute_force(w), rtol=0, atol=1e-12)


def test_golden_hand_example():
    with open(os.path.join(GOLDEN, "hand_example_gqa.json")) as f:
        g = json.load(f)
    D, P, NP = g["head_dim"], g["page_size"], g["num_pages"]
    pt = torch.tensor(g["page_table"], dtype=torch.int32)
    k = torch.full((NP, P, 1, D), float("nan"), dtype=torch.bfloat16)
    v = torch.full((NP, P, 1, D), float("nan"), dtype=torch.bfloat16)
    for t, (kt, vt) in enumerate(zip(g["k_tokens"], g["v_tokens"])):
        page = int(pt[0, t // P])
        k[page, t % P, 0] = torch.tensor(kt, dtype=torch.bfloat16)
        v[page, t % P, 0] = torch.tensor(vt, dtype=torch.bfloat16)
    w = workloads.Workload(name="golden", seed=0, q=torch.tensor(g["q"], dtype=torch.bfloat16), k_cache=k,
                           v_cache=v, page_table=pt, seq_lens=torch.tensor(g["seq_lens"], dtype=torch.int32),
                           scale=math.log(2.0))
    got = oracle.paged_decode(w)
    np.testing.assert_allclose(got, np.array(g["expected"]), rtol=0, atol=g["tolerance_abs"])
    for S in (1, 2, 3):
        np.testing.assert_allclose(oracle.paged_decode_split(w, S), np.array(g["expected"]), rtol=0,
                                   atol=g["tolerance_abs"])


def test_single_token_gives_v0():
    w = small(3, B=2, Hq=4, Hkv=2, D=32, P=8, lens=(1, 1), pool=6)
    got = oracle.paged_decode(w)
    for b in range(2):
        page = int(w.page_table[b, 0])
        for h in range(4):
            v0 = w.v_cache[page, 0, h // 2].to(torch.float64).numpy()
            assert np.array_equal(got[b, h], v0)
            assert torch.equal(oracle.round_bf16(got[b, h]), w.v_cache[page, 0, h // 2])


def test_zero_length_gives_zero():
    w = small(4, B=3, lens=(0, 9, 0))
    got = oracle.paged_decode(w)
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    assert np.all(got[1] != 0)
    assert np.all(oracle.paged_decode_split(w, 3)[[0, 2]] == 0)


def _mean_v(w, b, kvh):
    P = w.k_cache.shape[1]
    L = int(w.seq_lens[b])
    rows = [w.v_cache[int(w.page_table[b, t // P]), t % P, kvh].to(torch.float64) for t in range(L)]
    return torch.stack(rows).mean(0).numpy()


def test_constant_k_gives_mean_v():
    w = small(5, B=2, Hq=4, Hkv=2, D=32, P=4, lens=(13, 30))
    w.k_cache[:] = w.k_cache[0, 0, 0]  # every key row identical
    got = oracle.paged_decode(w)
    for b in range(2):
        for h in range(4):
            np.testing.assert_allclose(got[b, h], _mean_v(w, b, h // 2), rtol=0, atol=1e-12)


def test_zero_query_gives_mean_v():
    w = small(6, B=2, Hq=6, Hkv=3, D=16, P=4, lens=(7, 22))
    w.q.zero_()
    got = oracle.paged_decode(w)
    for b in range(2):
        for h in range(6):
            np.testing.assert_allclose(got[b, h], _mean_v(w, b, h // 2), rtol=0, atol=1e-12)


def test_huge_scale_unique_max_gives_v_argmax():
    w = small(7, B=2, Hq=2, Hkv=1, D=32, P=4, lens=(19, 11))
    P = 4
    # raw dot products, computed with numpy (not the oracle)
    kc = w.k_cache.to(torch.float64).numpy()
    vc = w.v_cache.to(torch.float64).numpy()
    qs = w.q.to(torch.float64).numpy()
    for b in range(2):
        L = int(w.seq_lens[b])
        for h in range(2):
            dots = np.array([qs[b, h] @ kc[int(w.page_table[b, t // P]), t % P, 0] for t in range(L)])
            order = np.argsort(dots)
            gap = dots[order[-1]] - dots[order[-2]]
            assert gap > 1e-3
            w.scale = 80.0 / gap  # runner-up weight <= e^-80
            got = oracle.paged_decode_rows(w, [(b, h)])[0]
            t = int(order[-1])
            np.testing.assert_allclose(got, vc[int(w.page_table[b, t // P]), t % P, 0], rtol=0, atol=1e-12)


def test_page_permutation_invariance():
    """Same logical sequences, other physical page placement: identical bits."""
    w = small(8, B=3, Hq=4, Hkv=2, D=32, P=4, lens=(5, 17, 12), pool=16)
    ref = oracle.paged_decode(w)
    rng = np.random.default_rng(1)
    perm = torch.from_numpy(rng.permutation(16))  # new placement: page p moves to perm[p]
    k2 = torch.empty_like(w.k_cache)
    v2 = torch.empty_like(w.v_cache)
    k2[perm] = w.k_cache
    v2[perm] = w.v_cache
    w2 = workloads.Workload(name="perm", seed=0, q=w.q, k_cache=k2, v_cache=v2,
                            page_table=perm[w.page_table.long()].to(torch.int32), seq_lens=w.seq_lens,
                            scale=w.scale)
    assert np.array_equal(oracle.paged_decode(w2), ref)


@pytest.mark.parametrize("layout", ["NHD", "HND"])
def test_split_invariance(layout):
    w = small(9, B=3, Hq=8, Hkv=2, D=32, P=4, lens=(37, 4, 64), layout=layout)
    ref = oracle.paged_decode(w)
    nmax = int(((w.seq_lens + 3) // 4).max())
    for S in (1, 2, 3, 7, nmax, nmax + 5):
        got = oracle.paged_decode_split(w, S)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_arbitrary_partition_invariance():
    w = small(10, B=2, Hq=4, Hkv=1, D=16, P=4, lens=(50, 23))
    ref = oracle.paged_decode(w)
    rng = np.random.default_rng(3)
    for b in range(2):
        L = int(w.seq_lens[b])
        for trial in range(5):
            cuts = sorted(rng.integers(0, L + 1, size=rng.integers(0, 6)).tolist())
            bounds = [0] + cuts + [L]  # may include empty chunks
            for h in range(4):
                got = oracle.paged_decode_chunks(w, b, h, bounds)
                np.testing.assert_allclose(got, ref[b, h], rtol=1e-12, atol=1e-13)


def test_partial_state_matches_definition():
    """(m, l, acc) of the whole range: acc / l is the output, m the max logit."""
    w = small(12, B=1, Hq=2, Hkv=1, D=16, P=4, lens=(21,))
    ref = oracle.paged_decode(w)
    acc, m, l = oracle.partial(w, 0, 1, 0, 21)
    np.testing.assert_allclose(acc / l, ref[0, 1], rtol=1e-12, atol=1e-13)
    acc0, m0, l0 = oracle.partial(w, 0, 1, 5, 5)
    assert m0 == -math.inf and l0 == 0 and not acc0.any()


def test_gqa_equals_mha_with_repeated_kv():
    w = small(13, B=2, Hq=8, Hkv=2, D=32, P=4, lens=(14, 27))
    g = 4
    w_mha = workloads.Workload(name="mha", seed=0, q=w.q, k_cache=w.k_cache.repeat_interleave(g, dim=2),
                               v_cache=w.v_cache.repeat_interleave(g, dim=2), page_table=w.page_table,
                               seq_lens=w.seq_lens, scale=w.scale)
    assert np.array_equal(oracle.paged_decode(w), oracle.paged_decode(w_mha))


def test_poisoned_slots_are_never_read():
    clean = small(14, B=3, Hq=4, Hkv=2, D=32, P=8, lens=(9, 16, 30), pool=10)
    dirty = small(14, B=3, Hq=4, Hkv=2, D=32, P=8, lens=(9, 16, 30), pool=10, poison=True)
    a = oracle.paged_decode(clean)
    b = oracle.paged_decode(dirty)
    assert np.isfinite(b).all()
    assert np.array_equal(a, b)


def test_rows_match_full():
    w = small(15, B=3, Hq=4, Hkv=2, D=16, P=4, lens=(6, 10, 3))
    full = oracle.paged_decode(w)
    rows = [(2, 3), (0, 0), (1, 2)]
    got = oracle.paged_decode_rows(w, rows)
    for i, (b, h) in enumerate(rows):
        assert np.array_equal(got[i], full[b, h])


def _bits(t):
    return int(t.view(torch.int16).item()) & 0xFFFF


def test_round_bf16_hand_examples():
    cases = [
        (1.0, 0x3F80),
        (-2.0, 0xC000),
        (1.0 + 2.0 ** -8, 0x3F80),          # tie between 1 and 1+2^-7 -> even (1)
        (1.0 + 3 * 2.0 ** -8, 0x3F82),      # tie between 1+2^-7 and 1+2^-6 -> even (1+2^-6)
        (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81),  # just above the tie -> up
        (0.0, 0x0000),
        (-0.0, 0x8000),
        (2.0 ** -133, 0x0001),              # smallest bf16 subnormal
        (2.0 ** -134, 0x0000),              # tie with zero -> even (0)
        (1.9921875 * 2.0 ** 127, 0x7F7F),   # largest finite bf16
        (1.99609375 * 2.0 ** 127, 0x7F80),  # rounds up past the largest finite -> +inf
        (math.inf, 0x7F80),
    ]
    for x, want in cases:
        assert _bits(oracle.round_bf16(np.array(x))) == want, (x, hex(want))
    assert math.isnan(float(oracle.round_bf16(np.array(math.nan))))


def test_round_bf16_matches_torch_on_float32_values():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(100000, generator=g) * torch.exp2(torch.randint(-20, 20, (100000,), generator=g).float())
    got = oracle.round_bf16(x.to(torch.float64).numpy())
    assert torch.equal(got.view(torch.int16), x.to(torch.bfloat16).view(torch.int16))
