"""GPU parity of the one-token streaming GEMV (tq_gemv, M = 1, G = 64 or 128,
K a multiple of 512 up to 4096, matrices too large for the pre-decode
kernel): lookup tables of one 512-column slice per CTA, the slices of a row
spread over a thread-block cluster of K / 512 CTAs.

fp32 outputs: max_n |gpu - oracle| <= 1e-3 * max_n |oracle| on the output
row; bf16 outputs: |gpu - oracle| <= 2e-2 + 2e-2 |oracle|; NaN outputs (rows
of W with a rejected group) must coincide, with the oracle's error bits.
Large matrices are built by repeating an oracle-packed block of rows (rows
are independent, so row n's expected output is the block's row n mod Nb).
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import (assert_close_bf16, assert_rows_close_f32, to_dev_bf16, to_dev_f16,
                          to_dev_u8, to_f64)

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def block(Nb, K, G, index):
    W = synthetic.weights(Nb, K, index=index, outlier_frac=1e-3)
    codes, scales, _ = oracle.quantize_pack(W, G)
    return codes, scales


def run(X, codes, scales, N, K, G, out_dtype=torch.float32):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = tq.gemv(to_dev_bf16(X), codes, scales, N, K, G, out_dtype=out_dtype, d_err=err)
    torch.cuda.synchronize()
    return to_f64(Y), int(err.item())


def tiled(Nb, reps, K, G, index):
    codes, scales = block(Nb, K, G, index)
    dc = to_dev_u8(codes).repeat(reps, 1, 1)
    ds = to_dev_f16(scales).repeat(reps, 1)
    return codes, scales, dc, ds


# (N, K, G): cluster sizes 1, 2, 4, 7 and 8, ragged row counts
SHAPES = [(16384, 1024, 128), (16384, 1024, 64), (16385, 1024, 128), (16391, 1024, 64),
          (40000, 512, 128), (40007, 512, 64), (9000, 2048, 64), (9001, 2048, 128),
          (4500, 3584, 128), (4501, 3584, 64), (4000, 4096, 64), (4097, 4096, 128)]


@pytest.mark.parametrize("N,K,G", SHAPES)
def test_stream_gemv_shapes(N, K, G):
    W = synthetic.weights(N, K, index=N % 1013 + K + G, outlier_frac=1e-3)
    codes, scales, _ = oracle.quantize_pack(W, G)
    X = synthetic.activations(1, K, offset=700)
    ref = oracle.linear(X, codes, scales, N, K, G)
    dc, ds = to_dev_u8(codes), to_dev_f16(scales)
    Y, e = run(X, dc, ds, N, K, G)
    assert_rows_close_f32(Y, ref)
    assert e == 0
    Yb, _ = run(X, dc, ds, N, K, G, torch.bfloat16)
    assert_close_bf16(Yb, ref)
    Y2, _ = run(X, dc, ds, N, K, G)
    assert np.array_equal(Y, Y2), "repeated launches differ"


@pytest.mark.parametrize("G", [64, 128])
def test_stream_gemv_ffn_stack_full_size(G):
    """The 48 gate/up projections of the 24-layer stack as one [172032 x 1024]
    matrix (the streaming benchmark's shape): four oracle-packed 3584-row
    projections repeated 12 times; every output compared."""
    K = 1024
    codes, scales = [], []
    for l in range(4):
        c, s, _ = oracle.quantize_pack(synthetic.ffn_matrix("gate", layer=l), G)
        codes.append(c)
        scales.append(s)
    codes, scales = np.concatenate(codes), np.concatenate(scales)
    Nb = codes.shape[0]
    N = 12 * Nb
    X = synthetic.activations(1, K, offset=701)
    ref_b = oracle.linear(X, codes, scales, Nb, K, G)
    ref = np.tile(ref_b, (1, 12))
    dc = to_dev_u8(codes).repeat(12, 1, 1)
    ds = to_dev_f16(scales).repeat(12, 1)
    Y, e = run(X, dc, ds, N, K, G)
    assert_rows_close_f32(Y, ref)
    assert e == 0


def test_stream_gemv_rounds():
    """More rows per cluster than its shared partial buffer holds (several
    rounds per cluster): 500,000 rows, K = 1024, G = 128."""
    K, G, Nb, reps = 1024, 128, 10000, 50
    codes, scales, dc, ds = tiled(Nb, reps, K, G, 31)
    X = synthetic.activations(1, K, offset=702)
    ref = np.tile(oracle.linear(X, codes, scales, Nb, K, G), (1, reps))
    Y, e = run(X, dc, ds, Nb * reps, K, G, torch.float32)
    assert_rows_close_f32(Y, ref)
    assert e == 0


@pytest.mark.parametrize("G", [64, 128])
def test_stream_gemv_rejected_groups(G):
    """Invalid bytes, bad padding, bad scales in both K slices and on the
    straddling code words give NaN outputs and the oracle's error bits; a
    zero group stays finite."""
    N, K = 16384, 1024
    codes, scales = block(N, K, G, 41)
    codes, scales = codes.copy(), scales.copy()
    B = (G + 4) // 5
    ng = K // G
    codes[5, 0, 0] = 250                     # invalid byte, first slice
    codes[77, ng - 1, B - 1] = 255           # invalid byte, last byte of the row
    codes[1000, ng // 2, B - 1] = 0          # padding digits 0, second slice
    codes[2001, 1, 0] = 243                  # smallest invalid value
    codes[16383, ng // 2 - 1, B - 1] = 242   # last byte of a first-slice group: digits 2 beyond G
    scales[3000, 2] = 0x7C00                 # Inf scale
    scales[4000, ng - 1] = 0x8000            # -0 scale
    scales[5000, 0] = 0x7E00                 # NaN scale
    scales[6000, 1] = 0                      # zero group: finite
    X = synthetic.activations(1, K, offset=703)
    ref = oracle.linear(X, codes, scales, N, K, G)
    _, e_ref = oracle.unpack_bf16(codes, scales, N, K, G)
    Y, e = run(X, to_dev_u8(codes), to_dev_f16(scales), N, K, G)
    assert_rows_close_f32(Y, ref)
    bad = [5, 77, 1000, 2001, 16383, 3000, 4000, 5000]
    assert np.all(np.isnan(Y[0, bad])) and np.isfinite(Y[0, 6000])
    assert e == e_ref and e != 0


def test_stream_gemv_every_byte_value():
    """Every byte value 0..255 at every code position of a slice: each row
    holds one byte value in all its positions (the padding rule then rejects
    the last bytes of most rows, as the oracle does)."""
    N, K, G = 16384, 1024, 128
    codes, scales = block(N, K, G, 42)
    codes = codes.copy()
    B = (G + 4) // 5
    rows = np.arange(256) * 61
    for v, r in enumerate(rows):
        codes[r, :, :] = v
        codes[r + 1, :, :B - 1] = v       # the last bytes stay canonical
    X = synthetic.activations(1, K, offset=704)
    ref = oracle.linear(X, codes, scales, N, K, G)
    _, e_ref = oracle.unpack_bf16(codes, scales, N, K, G)
    Y, e = run(X, to_dev_u8(codes), to_dev_f16(scales), N, K, G)
    assert_rows_close_f32(Y, ref)
    assert e == e_ref


@pytest.mark.parametrize("M", [2, 3, 4])
@pytest.mark.parametrize("G", [64, 128])
def test_stream_gemv_per_token(M, G):
    """2..4 tokens over a matrix of at least 48 M weights: one streaming
    launch per token row; every output compared."""
    N, K = 49159, 1024
    W = synthetic.weights(N, K, index=M + G, outlier_frac=1e-3)
    codes, scales, _ = oracle.quantize_pack(W, G)
    X = synthetic.activations(M, K, offset=11)
    ref = oracle.linear(X, codes, scales, N, K, G)
    dc, ds = to_dev_u8(codes), to_dev_f16(scales)
    Y, e = run(X, dc, ds, N, K, G)
    assert_rows_close_f32(Y, ref)
    assert e == 0
    Yb, _ = run(X, dc, ds, N, K, G, torch.bfloat16)
    assert_close_bf16(Yb, ref)

