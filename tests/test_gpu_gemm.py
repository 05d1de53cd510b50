"""GPU parity of tq_gemm (tensor-core prefill path) against the oracle.

fp32 outputs: max_n |gpu - oracle| <= 1e-3 * max_n |oracle| per output row;
bf16 outputs: |gpu - oracle| <= 2e-2 + 2e-2 |oracle|.  Full-size prefill
shapes are checked on sampled output rows computed one by one by the oracle.
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


def run(X, codes, scales, N, K, G, out_dtype):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = tq.gemm(to_dev_bf16(X), to_dev_u8(codes), to_dev_f16(scales), N, K, G, out_dtype=out_dtype, d_err=err)
    torch.cuda.synchronize()
    return to_f64(Y), int(err.item())


def check(X, W, G, dtypes=(torch.float32, torch.bfloat16), codes=None, scales=None):
    N, K = W.shape
    if codes is None:
        codes, scales, _ = oracle.quantize_pack(W, G)
    ref = oracle.linear(X, codes, scales, N, K, G)
    for dt in dtypes:
        Y, e = run(X, codes, scales, N, K, G, dt)
        assert e & tq.DERR_TIMEOUT == 0
        if dt == torch.float32:
            assert_rows_close_f32(Y, ref)
        else:
            assert_close_bf16(Y, ref)
    return ref


def test_tiny_workload():
    W, X, G = synthetic.tiny_case()
    ref = check(X, W, G)
    assert np.all(ref[:, :4] == 0)


@pytest.mark.parametrize("M,N,K,G", [(128, 256, 1024, 128), (1, 256, 640, 64), (7, 300, 1024, 64),
                                     (200, 1000, 1280, 128), (129, 257, 640, 64), (256, 512, 2048, 128),
                                     (64, 64, 192, 64)])
def test_shapes_and_tails(M, N, K, G):
    W = synthetic.weights(N, K, index=M + N, outlier_frac=1e-3)
    X = synthetic.activations(M, K)
    check(X, W, G)


def test_rejected_groups_give_nan_rows():
    G, N, K = 128, 300, 1024
    W = synthetic.weights(N, K, index=40)
    codes, scales, _ = oracle.quantize_pack(W, G)
    codes[3, 2, 4] = 250          # invalid byte
    codes[7, 1, 25] = 0           # padding digits 0
    scales[11, 5] = 0x7C00        # Inf scale
    scales[13, 0] = 0x8001        # negative scale
    scales[17, 3] = 0             # zero group: finite
    X = synthetic.activations(130, K)
    ref = check(X, W, G, codes=codes, scales=scales)
    assert np.all(np.isnan(ref[:, [3, 7, 11, 13]])) and np.all(np.isfinite(ref[:, 17]))
    _, e_ref = oracle.unpack_bf16(codes, scales, N, K, G)
    for M in (130, 16):  # prefill kernel; small-M kernel
        _, e = run(X[:M], codes, scales, N, K, G, torch.float32)
        assert e == e_ref


@pytest.mark.parametrize("G", [64, 128])
def test_every_code_byte(G):
    """All 243 valid bytes at every non-final byte position of a group, every
    canonical final byte, and the 13 invalid bytes (NaN rows), through the
    prefill kernel (M = 130) and the small-M kernel (M = 16)."""
    N, K = 520, 1024
    B = (G + 4) // 5
    real = G - 5 * (B - 1)  # digits of the final byte that hold weights
    finals = np.array([b for b in range(243)
                       if all((b // 3 ** i) % 3 == 1 for i in range(real, 5))], dtype=np.uint8)
    n = np.arange(N)[:, None, None]
    g = np.arange(K // G)[None, :, None]
    j = np.arange(B)[None, None, :]
    codes = ((n * B + g * 7 + j * 31) % 243).astype(np.uint8)
    codes[:, :, B - 1] = finals[(np.arange(N)[:, None] * 5 + np.arange(K // G)[None, :]) % finals.size]
    bad = list(range(507, 520))
    for i, r in enumerate(bad):
        codes[r, i % (K // G), (3 * i) % (B - 1)] = 243 + i
    scales = (synthetic.weights(N, K // G, index=9).astype(np.uint16) & 0x3FFF) | 0x0400
    X = synthetic.activations(130, K, offset=40)
    ref = oracle.linear(X, codes, scales, N, K, G)
    assert np.all(np.isnan(ref[:, bad])) and np.all(np.isfinite(ref[:, :507]))
    _, e_ref = oracle.unpack_bf16(codes, scales, N, K, G)
    for M in (130, 16):
        Y, e = run(X[:M], codes, scales, N, K, G, torch.float32)
        assert_rows_close_f32(Y, ref[:M])
        assert e == e_ref == tq.DERR_BYTE


def test_unsupported_group_size():
    W = synthetic.weights(64, 500, index=3)
    codes, scales, _ = oracle.quantize_pack(W, 100)
    X = synthetic.activations(4, 500)
    with pytest.raises(tq.TQError) as e:
        run(X, codes, scales, 64, 500, 100, torch.float32)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["up", "down"])
def test_prefill_full_size_sampled(name):
    """M=4096 prefill shapes, G=128, in the launch configuration the
    benchmark times; 32 sampled token rows checked against the oracle."""
    G, M = 128, synthetic.PREFILL_M
    W = synthetic.prefill_matrix(name)
    N, K = W.shape
    X = synthetic.activations(M, K)
    Wd = to_dev_bf16(W)
    codes, scales = tq.quantize_pack(Wd, G)
    del Wd
    Y = tq.gemm(to_dev_bf16(X), codes, scales, N, K, G, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = np.random.default_rng(7).choice(M, size=32, replace=False)
    c, s = codes.cpu().numpy(), scales.cpu().view(torch.int16).numpy().view(np.uint16)
    Wdec, _ = oracle.unpack_bf16(c, s, N, K, G)
    ref = oracle.matmul(X, Wdec, rows=rows)
    assert_close_bf16(to_f64(Y)[rows], ref)
