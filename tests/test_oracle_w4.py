"""Pins for the oracle's W4A16 affine decoding (a second weight format; only
its oracle is built so far, no kernels).

Source: tiny-llm "Week 2 Day 3: Quantize the Model", "Group-Wise Affine
Quantization", "Reconstruct a Stored Group", "Packed Storage Layout" and
"Revisit the Decode Roofline".  Expected values come from the page's packing
example and orientation example, its printed bytes per weight, brute force
over every code in every nibble, and exact rational sums.
"""
import os
from fractions import Fraction

import numpy as np
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x: float) -> int:
    return int(torch.tensor([x], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF


def bf16_frac(h: int) -> Fraction:
    return Fraction(float(torch.tensor([h], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).item()))


def one_group(word, s, b, G=8):
    return oracle.w4_dequant(np.array([[word]], dtype=np.uint32), np.array([[s]], dtype=np.uint16),
                             np.array([[b]], dtype=np.uint16), 1, G, G)[0]


def test_packing_example():
    """Eight codes [a..h] in one word: a in bits 0-3, ..., h in bits 28-31."""
    a_to_h = [1, 2, 3, 4, 5, 6, 7, 8]
    word = 0
    for i, q in enumerate(a_to_h):
        word |= q << (4 * i)
    assert word == 0x87654321
    assert one_group(word, bf16_bits(1.0), 0).tolist() == [float(q) for q in a_to_h]


def test_every_code_in_every_nibble():
    s, b = bf16_bits(0.375), bf16_bits(-1.25)
    for pos in range(8):
        for q in range(16):
            w = one_group(q << (4 * pos), s, b)
            want = [float(q * Fraction(3, 8) - Fraction(5, 4)) if i == pos else -1.25 for i in range(8)]
            assert w.tolist() == want, (pos, q)


def test_orientation_example():
    """Positive scale: code 0 at the bias, code 15 near 0.8; a negative scale
    with bias 0.8 reverses the order (the page's two parameter pairs)."""
    pos = one_group(0xF0000000, bf16_bits(0.0867), bf16_bits(-0.5))
    assert pos[0] == -0.5 and abs(pos[7] - 0.8) < 0.01
    neg = one_group(0xF0000000, bf16_bits(-0.0867), bf16_bits(0.8))
    assert neg[0] == float(bf16_frac(bf16_bits(0.8))) and abs(neg[7] + 0.5) < 0.01
    assert pos[7] > pos[0] and neg[7] < neg[0]


def test_bytes_per_weight_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "w4_bytes_per_weight.txt")) if not l.startswith("#")]
    for G, bpw in ((int(a), float(b)) for a, b in rows):
        N, K = 3, 4 * G
        codes_b = N * (K // 8) * 4          # uint32 words
        params_b = 2 * N * (K // G) * 2     # bf16 scale + bf16 bias per group
        assert (codes_b + params_b) / (N * K) == bpw


def test_groups_use_their_own_parameters():
    N, K, G = 3, 64, 16
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    scales = np.array([[bf16_bits(v) for v in rng.normal(0, 0.1, K // G)] for _ in range(N)], dtype=np.uint16)
    biases = np.array([[bf16_bits(v) for v in rng.normal(0, 1.0, K // G)] for _ in range(N)], dtype=np.uint16)
    W = oracle.w4_dequant(codes, scales, biases, N, K, G)
    for n in range(N):
        for k in range(K):
            q = (int(codes[n, k // 8]) >> (4 * (k % 8))) & 0xF
            want = q * bf16_frac(scales[n, k // G]) + bf16_frac(biases[n, k // G])
            assert Fraction(W[n, k]) == want, (n, k)


def test_linear_w4_exact_small():
    N, K, G, M = 4, 32, 16, 2
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    scales = np.array([[bf16_bits(v) for v in rng.normal(0, 0.1, K // G)] for _ in range(N)], dtype=np.uint16)
    biases = np.array([[bf16_bits(v) for v in rng.normal(0, 0.5, K // G)] for _ in range(N)], dtype=np.uint16)
    X = synthetic.activations(M, K)
    Y = oracle.linear_w4(X, codes, scales, biases, N, K, G)
    for m in range(M):
        for n in range(N):
            exact = sum(bf16_frac(int(X[m, k])) *
                        (((int(codes[n, k // 8]) >> (4 * (k % 8))) & 0xF) * bf16_frac(scales[n, k // G])
                         + bf16_frac(biases[n, k // G])) for k in range(K))
            assert abs(Y[m, n] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))
