"""Pins of the fp64 GEMV oracle against things other than itself: numpy's fp64
matmul (a library routine), closed forms (identity weights, one-hot inputs,
zero inputs), linearity in x, and the |x w| companion sum."""
import numpy as np
import pytest
import torch

import oracle
import workloads


def np_ref(x, w):
    return x.to(torch.float64).numpy() @ w.to(torch.float64).numpy().T


@pytest.mark.parametrize("M,N,K", [(1, 5, 16), (3, 64, 200), (8, 37, 1536), (2, 1, 8)])
def test_matches_numpy_matmul(M, N, K):
    c = workloads.gemv_case(M, N, K, seed=M * 100 + N)
    y, a = oracle.gemv(c.x, c.w)
    np.testing.assert_allclose(y, np_ref(c.x, c.w), rtol=1e-12, atol=1e-10)
    absref = np.abs(c.x.to(torch.float64).numpy()) @ np.abs(c.w.to(torch.float64).numpy()).T
    np.testing.assert_allclose(a, absref, rtol=1e-12)


def test_identity_weights_give_x():
    K = 48
    c = workloads.gemv_case(4, K, K, seed=3)
    eye = torch.eye(K, dtype=torch.bfloat16)
    y, _ = oracle.gemv(c.x, eye)
    assert np.array_equal(y, c.x.to(torch.float64).numpy())


def test_one_hot_inputs_select_weight_columns():
    c = workloads.gemv_case(3, 20, 64, seed=4)
    x = torch.zeros(3, 64, dtype=torch.bfloat16)
    for m, k in enumerate((0, 17, 63)):
        x[m, k] = 1.0
    y, _ = oracle.gemv(x, c.w)
    for m, k in enumerate((0, 17, 63)):
        assert np.array_equal(y[m], c.w[:, k].to(torch.float64).numpy())


def test_zero_input_gives_zero():
    c = workloads.gemv_case(2, 9, 32, seed=5)
    y, a = oracle.gemv(torch.zeros_like(c.x), c.w)
    assert not y.any() and not a.any()


def test_linearity_in_x():
    c = workloads.gemv_case(2, 30, 96, seed=6)
    y, _ = oracle.gemv(c.x, c.w)
    y2, _ = oracle.gemv((c.x.float() * 2).to(torch.bfloat16), c.w)  # x2 is exact in bf16
    assert np.array_equal(y2, 2 * y)
    xneg = -c.x
    yn, _ = oracle.gemv(xneg, c.w)
    assert np.array_equal(yn, -y)


def test_strided_rows():
    c = workloads.gemv_case(3, 11, 40, seed=8)
    xb = torch.zeros(3, 56, dtype=torch.bfloat16)
    xb[:, :40] = c.x
    wb = torch.zeros(11, 64, dtype=torch.bfloat16)
    wb[:, :40] = c.w
    y, _ = oracle.gemv(xb[:, :40], wb[:, :40])
    np.testing.assert_allclose(y, np_ref(c.x, c.w), rtol=1e-12, atol=1e-10)
