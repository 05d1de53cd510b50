"""GPU parity of tq_gemv (decode matmul, CUDA cores) against the oracle.

fp32 outputs: max_n |gpu - oracle| <= 1e-3 * max_n |oracle| per output row.
bf16 outputs: |gpu - oracle| <= 2e-2 + 2e-2 |oracle|.  NaN rows (rejected
groups) must coincide exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import (assert_close_bf16, assert_rows_close_f32, to_dev_bf16, to_dev_f16,
                          to_dev_u8, to_f64)

pytestmark = pytest.mark.gpu


def run(fn, X, codes, scales, N, K, G, out_dtype):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = fn(to_dev_bf16(X), to_dev_u8(codes), to_dev_f16(scales), N, K, G, out_dtype=out_dtype, d_err=err)
    torch.cuda.synchronize()
    return to_f64(Y), int(err.item())


def check(X, W, G, fn=tq.gemv, dtypes=(torch.float32, torch.bfloat16), codes=None, scales=None):
    N, K = W.shape
    if codes is None:
        codes, scales, _ = oracle.quantize_pack(W, G)
    ref = oracle.linear(X, codes, scales, N, K, G)
    _, e_ref = oracle.unpack_bf16(codes, scales, N, K, G)
    for dt in dtypes:
        Y, e = run(fn, X, codes, scales, N, K, G, dt)
        if dt == torch.float32:
            assert_rows_close_f32(Y, ref)
        else:
            assert_close_bf16(Y, ref)
        assert e == e_ref
    return ref


def test_tiny_workload():
    W, X, G = synthetic.tiny_case()
    ref = check(X, W, G)
    assert np.all(ref[:, :4] == 0)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("name", ["gate", "up", "down"])
def test_ffn_decode_full_size(name, G):
    W = synthetic.ffn_matrix(name)
    X = synthetic.activations(1, W.shape[1])
    check(X, W, G)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 9, 16, 33, 64])
@pytest.mark.parametrize("name", ["q", "gate", "down"])
def test_msweep_shapes(name, M):
    W = synthetic.msweep_matrix(name)
    X = synthetic.activations(M, W.shape[1])
    check(X, W, 128, dtypes=(torch.float32,))


@pytest.mark.parametrize("M", [1, 3])
@pytest.mark.parametrize("G", [1, 5, 8, 40, 64, 100, 128, 256, 4096])
def test_group_sizes_and_ragged_rows(G, M):
    K = G * max(2, 1024 // G)
    N = 77
    W = synthetic.weights(N, K, index=G + 50, outlier_frac=1e-3)
    X = synthetic.activations(M, K)
    check(X, W, G)


@pytest.mark.parametrize("M", [1, 2])
def test_rejected_groups_give_nan_rows(M):
    G, N, K = 64, 40, 512
    W = synthetic.weights(N, K, index=12)
    codes, scales, _ = oracle.quantize_pack(W, G)
    codes[3, 2, 4] = 250          # invalid byte
    codes[7, 1, 12] = 0           # padding digit 0
    scales[11, 5] = 0x7C00        # Inf scale
    scales[13, 0] = 0x8001        # negative scale
    scales[17, 3] = 0             # zero group: finite result
    X = synthetic.activations(M, K)
    ref = check(X, W, G, codes=codes, scales=scales)
    assert np.all(np.isnan(ref[:, [3, 7, 11, 13]])) and np.all(np.isfinite(ref[:, 17]))


@pytest.mark.parametrize("M", [1, 2])
def test_unaligned_codes_pointer(M):
    """Codes starting at an odd address are still served (the 16-bit code
    loads are not used then)."""
    G, N, K = 128, 300, 1024
    W = synthetic.weights(N, K, index=21)
    codes, scales, _ = oracle.quantize_pack(W, G)
    X = synthetic.activations(M, K)
    ref = oracle.linear(X, codes, scales, N, K, G)
    buf = torch.zeros(codes.size + 1, dtype=torch.uint8, device="cuda")
    buf[1:] = to_dev_u8(codes.reshape(-1))
    Y = tq.gemv(to_dev_bf16(X), buf[1:], to_dev_f16(scales), N, K, G, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_rows_close_f32(to_f64(Y), ref)


@pytest.mark.parametrize("N", [1, 7, 33, 3584 * 6])
def test_row_counts(N):
    G, K = 64, 1024
    W = synthetic.weights(N, K, index=N)
    X = synthetic.activations(1, K)
    check(X, W, G, dtypes=(torch.float32,))


@pytest.mark.parametrize("N,K,G", [(9477, 512, 64), (2000, 512, 32), (150, 4096, 256), (1500, 3072, 8),
                                   (700, 2048, 128), (300, 1024, 16)])
@pytest.mark.parametrize("M", [1, 4, 6, 8])
def test_predecode_row_batches(N, K, G, M):
    """One to eight tokens over matrices whose per-CTA rows fit in shared
    memory: more than eight row batches per CTA (8 rows, 4 rows from 5
    tokens), chunks split over two to eight warps, ragged last CTA, one or
    two CTAs per SM, tokens padded with zeros up to the kernel's 4 or 8
    (5..8 tokens with G a multiple of 64 take the tensor path instead)."""
    W = synthetic.weights(N, K, index=N + K)
    X = synthetic.activations(M, K)
    check(X, W, G)


@pytest.mark.parametrize("M", [5, 15, 16, 17, 31, 32, 48, 64])
@pytest.mark.parametrize("N,K,G", [(300, 1024, 128), (1536, 4096, 128), (257, 128, 64)])
def test_small_m_tensor_path(M, N, K, G):
    """5..64 tokens take the tensor-core small-M kernel (token tiles of 16, 32
    or 64, K split across a cluster)."""
    W = synthetic.weights(N, K, index=M * 7 + N)
    X = synthetic.activations(M, K)
    check(X, W, G)


@pytest.mark.parametrize("fn", [tq.gemv, tq.gemm, tq.gemv2])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_empty_sum_k0(fn, dt):
    """K = 0: every output is an empty sum, +0 (the output starts as NaN)."""
    M, N, G = 3, 77, 64
    X = torch.empty((M, 0), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((N, 0, 13), dtype=torch.uint8, device="cuda")
    scales = torch.empty((N, 0), dtype=torch.float16, device="cuda")
    Y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    fn(X, codes, scales, N, 0, G, out=Y)
    torch.cuda.synchronize()
    y = Y.float().cpu().numpy()
    assert np.all(y == 0) and not np.any(np.signbit(y))
