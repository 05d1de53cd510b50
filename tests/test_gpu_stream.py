"""GPU parity of the persistent small-M tensor-core path against the oracle.

Matrices with more 128-row tiles than half the SMs take it, from tq_gemm
for any M <= 64 and from tq_gemv for M >= 5 (3..4 when the pre-decode kernel
does not fit).  The decoded weights go to tensor memory as the MMA's A
operand.  Sampled token rows (first,
middle, last) are compared over every output column.  Tolerances as for the
other matmul paths: fp32 max_n |gpu - oracle| <= 1e-3 * max_n |oracle| per
row; bf16 |gpu - oracle| <= 2e-2 + 2e-2 |oracle|; NaN rows must coincide.
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

SHAPES = [(9600, 1024, 128), (19207, 1536, 64), (20000, 512, 256)]


@functools.lru_cache(maxsize=None)
def packed(N, K, G):
    W = synthetic.weights(N, K, index=N % 997 + G)
    codes, scales, _ = oracle.quantize_pack(W, G)
    return codes, scales


def run(fn, X, codes_dev, scales, N, K, G, out_dtype):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = fn(to_dev_bf16(X), codes_dev, to_dev_f16(scales), N, K, G, out_dtype=out_dtype, d_err=err)
    torch.cuda.synchronize()
    return to_f64(Y), int(err.item())


def sample_rows(M):
    return sorted({0, M // 2, M - 1})


@pytest.mark.parametrize("M", [1, 3, 8, 16, 17, 40, 64])
@pytest.mark.parametrize("N,K,G", SHAPES)
def test_stream_path(N, K, G, M):
    """More tiles than SMs (each CTA walks several tiles through the two TMEM
    accumulators), ragged last tile, token tiles of 16, 32 and 64."""
    codes, scales = packed(N, K, G)
    X = synthetic.activations(M, K)
    rows = sample_rows(M)
    ref = oracle.linear(X, codes, scales, N, K, G, rows=rows)
    fns = (tq.gemm, tq.gemv) if M >= 3 else (tq.gemm,)
    for fn in fns:
        Y, e = run(fn, X, to_dev_u8(codes), scales, N, K, G, torch.float32)
        assert_rows_close_f32(Y[rows], ref)
        assert e == 0
    Yb, _ = run(tq.gemm, X, to_dev_u8(codes), scales, N, K, G, torch.bfloat16)
    assert_close_bf16(Yb[rows], ref)


def test_stream_unaligned_codes_pointer():
    """Codes starting at an odd address: the per-row code windows are fetched
    from 16-byte aligned addresses inside the buffer and the edges byte by byte."""
    N, K, G, M = 9600, 1024, 128, 16
    codes, scales = packed(N, K, G)
    X = synthetic.activations(M, K)
    buf = torch.zeros(codes.size + 1, dtype=torch.uint8, device="cuda")
    buf[1:] = to_dev_u8(codes.reshape(-1))
    rows = sample_rows(M)
    ref = oracle.linear(X, codes, scales, N, K, G, rows=rows)
    Y, e = run(tq.gemm, X, buf[1:], scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y[rows], ref)
    assert e == 0


def test_stream_rejected_groups():
    """Rejected groups in several tiles give NaN output columns and their error bits."""
    N, K, G, M = 9600, 1024, 128, 8
    codes, scales = packed(N, K, G)
    codes, scales = codes.copy(), scales.copy()
    codes[5, 2, 4] = 250            # invalid byte
    codes[4000, 7, 25] = 0          # padding digit 0 in a last byte (G=128: 3 real digits)
    scales[9599, 1] = 0x7C00        # Inf scale, last row of the ragged tile
    scales[130, 0] = 0x8000         # -0 scale
    scales[7777, 3] = 0             # zero group: finite
    X = synthetic.activations(M, K)
    rows = sample_rows(M)
    ref = oracle.linear(X, codes, scales, N, K, G, rows=rows)
    _, e_ref = oracle.unpack_bf16(codes, scales, N, K, G)
    Y, e = run(tq.gemm, X, to_dev_u8(codes), scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y[rows], ref)
    assert np.all(np.isnan(Y[:, [5, 4000, 9599, 130]])) and np.all(np.isfinite(Y[:, 7777]))
    assert e == e_ref


@pytest.mark.parametrize("M", [8, 16])
def test_stream_path_ffn_stack_full_size(M):
    """The 48 gate/up projections of the 24-layer stack as one [172032 x 1024]
    matrix, G=128, through tq_gemv (each CTA walks about nine 128-row tiles):
    four oracle-packed 3584-row projections repeated 12 times; sampled token
    rows compared over every output column."""
    K, G = 1024, 128
    codes, scales = [], []
    for l in range(4):
        c, s_, _ = oracle.quantize_pack(synthetic.ffn_matrix("up", layer=l), G)
        codes.append(c)
        scales.append(s_)
    codes, scales = np.concatenate(codes), np.concatenate(scales)
    Nb = codes.shape[0]
    N = 12 * Nb
    X = synthetic.activations(M, K, offset=703)
    rows = sample_rows(M)
    ref = np.tile(oracle.linear(X, codes, scales, Nb, K, G, rows=rows), (1, 12))
    dc = to_dev_u8(codes).repeat(12, 1, 1)
    ds = to_dev_f16(scales).repeat(12, 1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = tq.gemv(to_dev_bf16(X), dc, ds, N, K, G, out_dtype=torch.float32, d_err=err)
    torch.cuda.synchronize()
    assert_rows_close_f32(to_f64(Y)[rows], ref)
    assert int(err.item()) == 0
