"""Pins for the oracle's matmul: Y[m, n] = sum_k X[m, k] * What[n, k].

Source: tiny-llm "Week 2 Day 3: Quantize the Model", "Mathematical
Formulation" (C = A B^T with B reconstructed per group) and "Computation
Flow".  Expected values come from exact rational arithmetic and from special
cases with closed forms (one-hot rows, all-ones rows, zero weights).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic


def frac_bf16_arr(a):
    v = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(torch.float64)
    return [[Fraction(x) for x in row] for row in v.numpy()]


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 8, 15), (2, 5, 24), (1, 4, 64)])
def test_matmul_bruteforce_rational(M, N, K):
    X = synthetic.normal_bf16((M, K), 1.0, seed=M * 100 + K)
    W = synthetic.normal_bf16((N, K), 0.02, seed=N * 100 + K)
    Y = oracle.matmul(X, W)
    fx, fw = frac_bf16_arr(X), frac_bf16_arr(W)
    for m in range(M):
        for n in range(N):
            exact = sum(a * b for a, b in zip(fx[m], fw[n]))
            assert abs(Fraction(Y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 45) + Fraction(1, 2 ** 200)


def test_matmul_points_agree_with_rows():
    X = synthetic.activations(5, 96)
    W = synthetic.weights(7, 96, index=2)
    Y = oracle.matmul(X, W)
    m = np.array([0, 4, 2, 2])
    n = np.array([6, 0, 3, 5])
    assert np.array_equal(oracle.matmul_points(X, W, m, n), Y[m, n])
    assert np.array_equal(oracle.matmul(X, W, rows=[3, 1]), Y[[3, 1]])


def test_matmul_one_hot_selects_a_column():
    W = synthetic.weights(9, 40, index=5)
    X = np.zeros((40, 40), dtype=np.uint16)
    X[np.arange(40), np.arange(40)] = 0x3F80  # bf16 1.0
    Y = oracle.matmul(X, W)
    ref = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(Y, ref.T)


def test_matmul_ones_gives_row_sums():
    W = synthetic.weights(6, 128, index=6)
    X = np.full((1, 128), 0x3F80, dtype=np.uint16)
    Y = oracle.matmul(X, W)
    for n, row in enumerate(frac_bf16_arr(W)):
        assert Fraction(Y[0, n]) == sum(row)   # 128 terms of 8-bit significands: exact in binary64


def test_layer_zero_rows_give_exact_zeros():
    W, X, G = synthetic.tiny_case()
    codes, scales, _ = oracle.quantize_pack(W, G)
    Y = oracle.linear(X, codes, scales, W.shape[0], W.shape[1], G)
    assert np.all(Y[:, :4] == 0.0)
    assert np.all(Y[:, 4:] != 0.0)


def test_layer_equals_grouped_formulation():
    """sum_g s_g * sum_j t_j x_j (the page's rearranged form with bias 0)
    equals the matmul with decoded weights, exactly in rationals."""
    G, N, K = 10, 3, 40
    W = synthetic.weights(N, K, index=8)
    X = synthetic.activations(2, K)
    codes, scales, _ = oracle.quantize_pack(W, G)
    Y = oracle.linear(X, codes, scales, N, K, G)
    fx = frac_bf16_arr(X)
    for n in range(N):
        for m in range(2):
            acc = Fraction(0)
            for g in range(K // G):
                s = scales[n, g]
                sb = torch.tensor([float(np.array([s], np.uint16).view(np.float16)[0])],
                                  dtype=torch.float32).to(torch.bfloat16).to(torch.float64).item()
                inner = Fraction(0)
                for j in range(G):
                    b = int(codes[n, g, j // 5])
                    t = (b // 3 ** (j % 5)) % 3 - 1
                    inner += t * fx[m][g * G + j]
                acc += Fraction(sb) * inner
            assert Fraction(Y[m, n]) == acc


def test_invalid_group_poisons_its_row():
    W = synthetic.weights(4, 128, index=1)
    codes, scales, _ = oracle.quantize_pack(W, 64)
    codes[2, 1, 5] = 250
    X = synthetic.activations(3, 128)
    Y = oracle.linear(X, codes, scales, 4, 128, 64)
    assert np.all(np.isnan(Y[:, 2]))
    assert np.all(np.isfinite(np.delete(Y, 2, axis=1)))
