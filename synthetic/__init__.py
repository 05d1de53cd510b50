"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the method (no scale, trit, codec or matmul
step): it only draws seeded random matrices with the shapes and value
distributions of the workloads and rounds them to bf16 bit patterns with
torch's round-to-nearest-even conversion.  Both the CUDA path and the oracle
consume what it returns, so they always see identical bits.

Workloads (the matrix shapes follow the pages' models):
  * tiny:     one 256 x 640 weight matrix (out x in), G=64, W ~ N(0, 0.02) with
              rows 0..3 set to exact zeros, X ~ N(0, 1), M=1.
  * ffn:      Qwen3.5-0.8B-shaped FFN projections, gate/up 3584 x 1024 and
              down 1024 x 3584, W ~ N(0, 0.02) with 0.1% of the entries
              (uniform positions) scaled by 10, X ~ N(0, 1).
  * stack:    24 layers x (gate, up, down) of those shapes: 72 matrices,
              264,241,152 weights, W ~ N(0, 0.02).
  * msweep:   a 28-layer, width-1536 Llama-style stack: q/o 1536 x 1536,
              gate/up 4096 x 1536, down 1536 x 4096; G=128; M in 1..64.
  * prefill:  M=4096 tokens, K=4096 -> N=14336 and K=14336 -> N=4096, G=128.
Seeds: weights 1000 + matrix index, activations 2000 + M (+ a per-use offset),
outlier positions 3000 + matrix index.
"""
from __future__ import annotations

import numpy as np
import torch

SEED_W = 1000
SEED_X = 2000
SEED_OUTLIER = 3000

FFN_SHAPES = {"gate": (3584, 1024), "up": (3584, 1024), "down": (1024, 3584)}
MSWEEP_SHAPES = {"q": (1536, 1536), "o": (1536, 1536), "gate": (4096, 1536),
                 "up": (4096, 1536), "down": (1536, 4096)}
PREFILL_SHAPES = {"up": (14336, 4096), "down": (4096, 14336)}  # (N out, K in)
PREFILL_M = 4096


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), round to nearest even (torch)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def normal_bf16(shape, sigma: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return to_bf16_bits(a)


def weights(N: int, K: int, index: int = 0, sigma: float = 0.02,
            outlier_frac: float = 0.0, outlier_mult: float = 10.0) -> np.ndarray:
    """[N, K] bf16 bits ~ N(0, sigma); optionally a fraction of entries scaled."""
    rng = np.random.default_rng(SEED_W + index)
    a = rng.standard_normal(size=(N, K), dtype=np.float32)
    a *= np.float32(sigma)
    if outlier_frac > 0:
        orng = np.random.default_rng(SEED_OUTLIER + index)
        cnt = int(round(outlier_frac * N * K))
        pos = orng.choice(N * K, size=cnt, replace=False)
        a.reshape(-1)[pos] *= np.float32(outlier_mult)
    return to_bf16_bits(a)


def activations(M: int, K: int, offset: int = 0) -> np.ndarray:
    """[M, K] bf16 bits ~ N(0, 1)."""
    return normal_bf16((M, K), 1.0, SEED_X + M + offset)


def tiny_case():
    """(W [256, 640], X [1, 640], G=64) with rows 0..3 of W exactly zero."""
    W = weights(256, 640, index=0)
    W[0:4, :] = 0
    X = activations(1, 640)
    return W, X, 64


def ffn_matrix(name: str, layer: int = 0, outliers: bool = True) -> np.ndarray:
    N, K = FFN_SHAPES[name]
    idx = 3 * layer + ["gate", "up", "down"].index(name)
    return weights(N, K, index=idx, outlier_frac=1e-3 if outliers else 0.0)


def msweep_matrix(name: str, layer: int = 0) -> np.ndarray:
    N, K = MSWEEP_SHAPES[name]
    idx = 100 + 5 * layer + list(MSWEEP_SHAPES).index(name)
    return weights(N, K, index=idx)


def prefill_matrix(name: str) -> np.ndarray:
    N, K = PREFILL_SHAPES[name]
    return weights(N, K, index=900 + list(PREFILL_SHAPES).index(name))


def random_bf16_bits(shape, seed: int, finite_only: bool = True) -> np.ndarray:
    """Uniformly random bf16 bit patterns (every exponent), for edge-case tests."""
    rng = np.random.default_rng(seed)
    b = rng.integers(0, 1 << 16, size=shape, dtype=np.uint32).astype(np.uint16)
    if finite_only:
        bad = (b & 0x7F80) == 0x7F80
        b[bad] &= 0xBFFF  # clear the top exponent bit: a finite pattern
    return b


def w4_params(N: int, K: int, G: int, index: int = 0):
    """Seeded W4A16 affine parameters of an [N, K] matrix: codes uint32
    [N, K/8] (eight uniform 4-bit codes per word), scales and biases as bf16
    bit patterns [N, K/G].  Magnitudes follow an affine 4-bit quantization
    of N(0, 0.02) weights over groups of G (scale ~ range / 15, bias ~ the
    group minimum); scales carry random signs."""
    rng = np.random.default_rng(SEED_W + 5000 + index)
    codes = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    mag = rng.uniform(0.004, 0.009, size=(N, K // G)).astype(np.float32)
    sign = np.where(rng.random(size=(N, K // G)) < 0.5, -1.0, 1.0).astype(np.float32)
    scales = to_bf16_bits(mag * sign)
    biases = to_bf16_bits(rng.normal(0.0, 0.05, size=(N, K // G)).astype(np.float32))
    return codes, scales, biases
