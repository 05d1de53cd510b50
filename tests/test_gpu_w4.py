"""GPU parity of tq_w4_gemv (the W4A16 affine format, CUDA cores) against the
oracle's binary64 reconstruction w = q * s + b and matmul.

fp32 outputs: max_n |gpu - oracle| <= 1e-3 * max_n |oracle| per output row;
bf16 outputs: |gpu - oracle| <= 2e-2 + 2e-2 |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import assert_close_bf16, assert_rows_close_f32, to_dev_bf16, to_f64

pytestmark = pytest.mark.gpu


def dev_params(codes, scales, biases):
    c = torch.from_numpy(codes.view(np.int32)).cuda()
    return c, to_dev_bf16(scales), to_dev_bf16(biases)


def check(N, K, G, M, index=0, dtypes=(torch.float32, torch.bfloat16)):
    codes, scales, biases = synthetic.w4_params(N, K, G, index=index)
    X = synthetic.activations(M, K, offset=800)
    ref = oracle.linear_w4(X, codes, scales, biases, N, K, G)
    dc, ds, db = dev_params(codes, scales, biases)
    for dt in dtypes:
        Y = tq.w4_gemv(to_dev_bf16(X), dc, ds, db, N, K, G, out_dtype=dt)
        torch.cuda.synchronize()
        if dt == torch.float32:
            assert_rows_close_f32(to_f64(Y), ref)
        else:
            assert_close_bf16(to_f64(Y), ref)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 11])
@pytest.mark.parametrize("N,K,G", [(3584, 1024, 128), (1024, 3584, 128), (1536, 1536, 64), (4096, 1536, 32)])
def test_w4_gemv_shapes(N, K, G, M):
    """Streaming kernel: one to four 32-column chunks per lane and row, one to
    eight tokens per launch, two launches past eight tokens."""
    check(N, K, G, M, index=N + K + G)


@pytest.mark.parametrize("N,K,G", [(77, 4096, 128), (9, 96, 32), (2001, 512, 512)])
def test_w4_gemv_ragged_rows(N, K, G):
    check(N, K, G, 1, index=N)


@pytest.mark.parametrize("N,K,G", [(300, 1024, 8), (129, 960, 48), (64, 8192, 128), (50, 1000, 40)])
@pytest.mark.parametrize("M", [1, 5])
def test_w4_gemv_generic_shapes(N, K, G, M):
    """Group sizes that are not multiples of 32, and K beyond the streaming
    kernel's 4096: the one-warp-per-row kernel."""
    check(N, K, G, M, index=G + 7)


def test_w4_gemv_every_code_value():
    """Each code value 0..15 in every nibble position: rows of constant words."""
    N, K, G = 64, 1024, 128
    codes, scales, biases = synthetic.w4_params(N, K, G, index=3)
    for q in range(16):
        codes[q] = np.uint32(sum(q << (4 * k) for k in range(8)))
    X = synthetic.activations(1, K, offset=801)
    ref = oracle.linear_w4(X, codes, scales, biases, N, K, G)
    dc, ds, db = dev_params(codes, scales, biases)
    Y = tq.w4_gemv(to_dev_bf16(X), dc, ds, db, N, K, G, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_rows_close_f32(to_f64(Y), ref)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("K", [256, 512, 768, 1024, 1280, 1536, 1792, 2048])
def test_w4_gemv_stream(K, G):
    """One token over 16 M weights and more: the streaming lookup-table kernel
    (tables of 256 columns per CTA, K / 256 CTAs per cluster, one to eight),
    the last cluster's rows ragged."""
    N = (16 << 20) // K + 37
    check(N, K, G, 1, index=K + 3 * G)


@pytest.mark.parametrize("M", [2, 3, 4])
@pytest.mark.parametrize("N,K,G", [(24593, 512, 128), (49157, 256, 64)])
def test_w4_gemv_stream_tokens(N, K, G, M):
    """2..4 tokens at K <= 512 over 12 Mi weights and more: one streaming
    launch per token."""
    check(N, K, G, M, index=M + K)


def test_w4_gemv_stream_tokens_large():
    """Two tokens over 96 Mi weights and more (K = 1024): one streaming launch
    per token."""
    check(98317, 1024, 128, 2, index=17, dtypes=(torch.bfloat16,))


@pytest.mark.parametrize("M", [1, 2])
def test_w4_gemv_stream_full_size_sampled(M):
    """The benchmark's workload: the 24-layer gate/up-shaped stack as one
    [172032 x 1024] W4A16 matrix, G=128 (4-CTA clusters), one and two tokens
    (one streaming launch per token); 512 sampled output columns against the
    oracle on the same rows."""
    N, K, G = 48 * 3584, 1024, 128
    codes, scales, biases = synthetic.w4_params(N, K, G, index=41)
    X = synthetic.activations(M, K, offset=805)
    dc, ds, db = dev_params(codes, scales, biases)
    Y = tq.w4_gemv(to_dev_bf16(X), dc, ds, db, N, K, G, out_dtype=torch.float32)
    torch.cuda.synchronize()
    cols = np.random.default_rng(1).choice(N, size=512, replace=False)
    ref = oracle.linear_w4(X, codes[cols], scales[cols], biases[cols], len(cols), K, G)
    assert_rows_close_f32(to_f64(Y)[:, cols], ref)


def test_w4_gemv_stream_every_byte():
    """Every code byte (two nibbles) in every byte position of the tables:
    row n, word w, byte i holds (n + 8 w + i) mod 256."""
    N, K, G = 16411, 1024, 128
    codes, scales, biases = synthetic.w4_params(N, K, G, index=5)
    n = np.arange(N, dtype=np.uint32)[:, None, None]
    w = np.arange(K // 8, dtype=np.uint32)[None, :, None]
    i = np.arange(4, dtype=np.uint32)[None, None, :]
    byte = (n + 8 * w + i) % 256
    codes = (byte << (8 * i)).sum(axis=2).astype(np.uint32)
    X = synthetic.activations(1, K, offset=802)
    ref = oracle.linear_w4(X, codes, scales, biases, N, K, G)
    dc, ds, db = dev_params(codes, scales, biases)
    Y = tq.w4_gemv(to_dev_bf16(X), dc, ds, db, N, K, G, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_rows_close_f32(to_f64(Y), ref)


def test_w4_gemv_stream_unaligned_operands():
    """Scales and biases views that start 2 bytes in (not 4-byte aligned): the
    streaming kernel declines and the row kernel answers."""
    N, K, G = 16411, 1024, 128
    codes, scales, biases = synthetic.w4_params(N, K, G, index=6)
    X = synthetic.activations(1, K, offset=803)
    ref = oracle.linear_w4(X, codes, scales, biases, N, K, G)
    dc, ds, db = dev_params(codes, scales, biases)
    flat_s = torch.empty(ds.numel() + 1, dtype=torch.bfloat16, device="cuda")
    flat_s[1:] = ds.reshape(-1)
    flat_b = torch.empty(db.numel() + 1, dtype=torch.bfloat16, device="cuda")
    flat_b[1:] = db.reshape(-1)
    Y = tq.w4_gemv(to_dev_bf16(X), dc, flat_s[1:].view(N, K // G), flat_b[1:].view(N, K // G), N, K, G,
                   out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_rows_close_f32(to_f64(Y), ref)


@pytest.mark.parametrize("M", [5, 16, 40])
@pytest.mark.parametrize("N,K,G", [(16411, 1024, 128), (12007, 2048, 64)])
def test_w4_gemv_persistent_tensor_path(N, K, G, M):
    """5..64 tokens on matrices with more 128-row tiles than half the SMs:
    the persistent small-M tensor kernel (hi and lo bf16 terms of each weight
    in tensor memory), token tiles of 16 and 64, ragged last tile."""
    check(N, K, G, M, index=N + M, dtypes=(torch.float32,))


def test_w4_gemv_persistent_unaligned_codes():
    """Codes 4 bytes past a 16-byte boundary: the persistent tensor kernel
    (16-byte code windows) declines and the CUDA-core kernel answers."""
    N, K, G, M = 16411, 1024, 128, 8
    codes, scales, biases = synthetic.w4_params(N, K, G, index=9)
    X = synthetic.activations(M, K, offset=806)
    ref = oracle.linear_w4(X, codes, scales, biases, N, K, G)
    dc, ds, db = dev_params(codes, scales, biases)
    flat = torch.empty(dc.numel() + 1, dtype=torch.int32, device="cuda")
    flat[1:] = dc.reshape(-1)
    Y = tq.w4_gemv(to_dev_bf16(X), flat[1:].view(N, K // 8), ds, db, N, K, G, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_rows_close_f32(to_f64(Y), ref)


@pytest.mark.parametrize("M", [1, 16, 256, 300])
@pytest.mark.parametrize("N,K,G", [(512, 1024, 128), (1000, 4096, 64), (4096, 1024, 128), (130, 2048, 256)])
def test_w4_gemm_tensor_cores(N, K, G, M):
    """tq_w4_gemm: the W4 weights as two bf16 terms (hi + remainder) on the
    tensor cores; the fp32 per-row tolerance holds on every output."""
    codes, scales, biases = synthetic.w4_params(N, K, G, index=N + 3 * K + G)
    X = synthetic.activations(M, K, offset=802)
    ref = oracle.linear_w4(X, codes, scales, biases, N, K, G)
    dc, ds, db = dev_params(codes, scales, biases)
    for dt in (torch.float32, torch.bfloat16):
        Y = tq.w4_gemm(to_dev_bf16(X), dc, ds, db, N, K, G, out_dtype=dt)
        torch.cuda.synchronize()
        if dt == torch.float32:
            assert_rows_close_f32(to_f64(Y), ref)
        else:
            assert_close_bf16(to_f64(Y), ref)


def test_w4_gemm_unsupported_group_size():
    N, K, G = 64, 1024, 32
    codes, scales, biases = synthetic.w4_params(N, K, G, index=5)
    dc, ds, db = dev_params(codes, scales, biases)
    with pytest.raises(tq.TQError, match="UNSUPPORTED"):
        tq.w4_gemm(to_dev_bf16(synthetic.activations(4, K)), dc, ds, db, N, K, G)
