"""GPU parity of the 2-bit ternary format (four codes per byte) against the oracle.

tq2_quantize_pack and tq2_unpack_bf16: bit-exact on scales, code bytes,
decoded bf16 weights and error bits.  tq2_gemv: the fused matmul's
tolerances (fp32 max_n |gpu - oracle| <= 1e-3 * max_n |oracle| per row; bf16
|gpu - oracle| <= 2e-2 + 2e-2 |oracle|; NaN rows must coincide) and the
oracle's error bits.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import (assert_close_bf16, assert_rows_close_f32, bits_u16, to_dev_bf16, to_dev_f16,
                          to_dev_u8, to_f64)

pytestmark = pytest.mark.gpu


def gpu_pack2(W_bits, G):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = tq.quantize_pack2(to_dev_bf16(W_bits), G, d_err=err)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), bits_u16(scales), int(err.item())


def gpu_unpack2(codes, scales_bits, N, K, G):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tq.unpack2_bf16(to_dev_u8(codes), to_dev_f16(scales_bits), N, K, G, d_err=err)
    torch.cuda.synchronize()
    return bits_u16(out), int(err.item())


def check_pack2(W_bits, G):
    c_ref, s_ref, e_ref = oracle.quantize_pack2(W_bits, G)
    c, s, e = gpu_pack2(W_bits, G)
    assert np.array_equal(s.reshape(s_ref.shape), s_ref), np.argwhere(s.reshape(s_ref.shape) != s_ref)[:8]
    assert np.array_equal(c.reshape(c_ref.shape), c_ref), np.argwhere(c.reshape(c_ref.shape) != c_ref)[:8]
    assert e == e_ref
    return c_ref, s_ref


def check_unpack2(codes, scales, N, K, G):
    w_ref, e_ref = oracle.unpack2_bf16(codes, scales, N, K, G)
    w, e = gpu_unpack2(codes, scales, N, K, G)
    assert np.array_equal(w.reshape(w_ref.shape), w_ref), np.argwhere(w.reshape(w_ref.shape) != w_ref)[:8]
    assert e == e_ref


@pytest.mark.parametrize("G", [8, 16, 32, 64, 128, 256, 6, 12, 48, 100])
def test_group_sizes(G):
    """Group kernels (G = 8..128), the generic kernel (others), word and
    generic unpack; ragged row counts; every exponent, zero and subnormal
    groups, non-finite weights and overflowing means."""
    K = G * max(2, 512 // G)
    N = 37
    W = synthetic.weights(N, K, index=G, outlier_frac=0.01)
    W[5] = synthetic.random_bf16_bits(K, seed=G)
    W[6] = 0
    W[7, : K // 2] = 0x0001
    W[8, 1] = 0x7F80
    W[9, :G] = 0x7F7F
    codes, scales = check_pack2(W, G)
    check_unpack2(codes, scales, N, K, G)


@pytest.mark.parametrize("G", [64, 128])
def test_ffn_full_size(G):
    W = synthetic.ffn_matrix("gate")
    codes, scales = check_pack2(W, G)
    check_unpack2(codes, scales, W.shape[0], W.shape[1], G)


@pytest.mark.parametrize("G", [16, 64, 128, 256, 10])
def test_unpack2_rejections(G):
    """Code 3 anywhere, padding codes other than 1, rejected scales and zero
    groups; a rejected group is NaN as a whole, the error bits are the oracle's."""
    N, K = 50, 4 * G
    W = synthetic.weights(N, K, index=5)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    rng = np.random.default_rng(G)
    B = codes.shape[2]
    for n in range(0, N, 3):
        g = rng.integers(0, K // G)
        kind = n % 4
        if kind == 0:
            q, i = rng.integers(0, B), rng.integers(0, 4)
            codes[n, g, q] |= 3 << (2 * i)
        elif kind == 1 and G % 4:
            codes[n, g, B - 1] &= 0x3F  # last padding code 0
        elif kind == 2:
            scales[n, g] = [0x7C00, 0xFC00, 0x7E01, 0x8001][n % 4]
        else:
            scales[n, g] = 0
    check_unpack2(codes, scales, N, K, G)


def run_gemv2(X, codes, scales, N, K, G, out_dtype):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = tq.gemv2(to_dev_bf16(X), to_dev_u8(codes), to_dev_f16(scales), N, K, G, out_dtype=out_dtype, d_err=err)
    torch.cuda.synchronize()
    return to_f64(Y), int(err.item())


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 11])
@pytest.mark.parametrize("N,K,G", [(3584, 1024, 64), (1024, 3584, 128), (1037, 1152, 128), (301, 1040, 16),
                                   (130, 4096, 256), (77, 2048, 32), (300, 1024, 16)])
def test_gemv2(N, K, G, M):
    """Token counts 1..11 (two launches past 8), ragged row batches and code
    words per row that are not multiples of 32 lanes; fp32 and bf16 outputs.
    K a multiple of 512 takes the pre-decode kernel up to 4 tokens (8 at
    G < 64: one, two and four code words per decode lane), other K the
    CUDA-core kernel, 5+ tokens at G % 64 == 0 the tensor path."""
    W = synthetic.weights(N, K, index=N + G)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    X = synthetic.activations(M, K)
    ref = oracle.linear2(X, codes, scales, N, K, G)
    Y, e = run_gemv2(X, codes, scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y, ref)
    assert e == 0
    Yb, _ = run_gemv2(X, codes, scales, N, K, G, torch.bfloat16)
    assert_close_bf16(Yb, ref)


def test_gemv2_rejected_groups():
    N, K, G, M = 515, 1024, 64, 3
    W = synthetic.weights(N, K, index=11)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    codes[5, 2, 7] |= 0xC0      # code 3
    scales[130, 0] = 0x7C00     # Inf scale
    scales[514, 15] = 0x8000    # -0 scale, last row
    scales[77, 3] = 0           # zero group: finite
    X = synthetic.activations(M, K)
    ref = oracle.linear2(X, codes, scales, N, K, G)
    _, e_ref = oracle.unpack2_bf16(codes, scales, N, K, G)
    Y, e = run_gemv2(X, codes, scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y, ref)
    assert np.all(np.isnan(Y[:, [5, 130, 514]])) and np.all(np.isfinite(Y[:, 77]))
    assert e == e_ref == tq.DERR_BYTE | tq.DERR_SCALE


def test_gemv2_stack_full_size_sampled():
    """The 24-layer gate/up stack as one [172032 x 1024] matrix, G=128, M=1
    (the streaming decode workload), packed on the GPU; sampled output
    columns against the oracle."""
    N, K, G = 48 * 3584, 1024, 128
    W = np.concatenate([synthetic.ffn_matrix(n, layer=l, outliers=False)
                        for l in range(24) for n in ("gate", "up")])
    c, s, e = gpu_pack2(W, G)
    assert e == 0
    X = synthetic.activations(1, K)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = tq.gemv2(to_dev_bf16(X), to_dev_u8(c), to_dev_f16(s), N, K, G, out_dtype=torch.float32, d_err=err)
    torch.cuda.synchronize()
    cols = np.random.default_rng(0).choice(N, size=512, replace=False)
    c_ref, s_ref, _ = oracle.quantize_pack2(W[cols], G)
    assert np.array_equal(c.reshape(N, K // G, -1)[cols], c_ref)
    ref = oracle.linear2(X, c_ref, s_ref, len(cols), K, G)
    assert_rows_close_f32(to_f64(Y)[:, cols], ref)
    assert int(err.item()) == 0


# M = 1, G in {64, 128}, K a multiple of 512 up to 4096: the streaming
# lookup-table kernel (cluster sizes 1..8, ragged row counts)
STREAM2_SHAPES = [(16385, 512, 128), (16391, 1024, 64), (9001, 2048, 128), (3000, 1536, 64),
                  (4501, 3584, 64), (4097, 4096, 128), (257, 2560, 128), (7000, 3072, 64)]


@pytest.mark.parametrize("N,K,G", STREAM2_SHAPES)
def test_gemv2_stream_shapes(N, K, G):
    W = synthetic.weights(N, K, index=N % 997 + G, outlier_frac=1e-3)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    X = synthetic.activations(1, K, offset=300)
    ref = oracle.linear2(X, codes, scales, N, K, G)
    Y, e = run_gemv2(X, codes, scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y, ref)
    assert e == 0
    Yb, _ = run_gemv2(X, codes, scales, N, K, G, torch.bfloat16)
    assert_close_bf16(Yb, ref)
    Y2, _ = run_gemv2(X, codes, scales, N, K, G, torch.float32)
    assert np.array_equal(Y, Y2), "repeated launches differ"


@pytest.mark.parametrize("G", [64, 128])
def test_gemv2_stream_every_valid_byte(G):
    """Every one of the 81 valid code bytes at every byte position of a
    512-column slice (both K slices of a 2-CTA cluster), in rows that run
    past a warp's share and a cluster's share."""
    N, K = 9001, 1024
    B = G // 4
    valid = np.array([b for b in range(256) if all((b >> (2 * i)) & 3 != 3 for i in range(4))], dtype=np.uint8)
    assert valid.size == 81
    n = np.arange(N)[:, None, None]
    g = np.arange(K // G)[None, :, None]
    j = np.arange(B)[None, None, :]
    codes = valid[(n * 7 + g * B + j * 11) % 81].astype(np.uint8)
    scales = synthetic.weights(N, K // G, index=5).astype(np.uint16) & 0x3FFF  # positive finite binary16
    X = synthetic.activations(1, K, offset=900)
    ref = oracle.linear2(X, codes, scales, N, K, G)
    Y, e = run_gemv2(X, codes, scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y, ref)
    assert e == 0


@pytest.mark.parametrize("G", [64, 128])
def test_gemv2_stream_rejected_groups(G):
    """Code 3 in each byte lane of a word, in both K slices and in the first
    and last rows; Inf, NaN and -0 scales; zero groups stay finite."""
    N, K = 20000, 1024
    W = synthetic.weights(N, K, index=G + 3)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    B = G // 4
    bad_rows = []
    for i, (n, byte) in enumerate([(0, 0), (1, 5), (777, 9), (4096, B - 1), (12345, 3), (N - 1, 7)]):
        grp = i % (K // G)
        codes[n, grp, byte % B] |= 0x03 << (2 * (i % 4))
        bad_rows.append(n)
    scales[130, 0] = 0x7C00
    scales[9999, K // G - 1] = 0x7E00
    scales[N - 2, 1] = 0x8000
    scales[77, 3] = 0
    bad_rows += [130, 9999, N - 2]
    X = synthetic.activations(1, K)
    ref = oracle.linear2(X, codes, scales, N, K, G)
    _, e_ref = oracle.unpack2_bf16(codes, scales, N, K, G)
    Y, e = run_gemv2(X, codes, scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y, ref)
    assert np.all(np.isnan(Y[:, bad_rows])) and np.all(np.isfinite(Y[:, 77]))
    assert e == e_ref == tq.DERR_BYTE | tq.DERR_SCALE


@pytest.mark.parametrize("M", [2, 4])
@pytest.mark.parametrize("G", [64, 128])
def test_gemv2_stream_per_token(M, G):
    """2..4 tokens over a matrix of at least 48 M weights: one streaming
    launch per token row."""
    N, K = 24593, 2048
    W = synthetic.weights(N, K, index=M * G)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    X = synthetic.activations(M, K, offset=5)
    ref = oracle.linear2(X, codes, scales, N, K, G)
    Y, e = run_gemv2(X, codes, scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y, ref)
    assert e == 0


def test_gemv2_unsupported_group_size():
    N, K, G = 64, 480, 48
    W = synthetic.weights(N, K, index=1)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    with pytest.raises(tq.TQError, match="UNSUPPORTED"):
        run_gemv2(synthetic.activations(1, K), codes, scales, N, K, G, torch.float32)


def run_mm2(fn, X, codes, scales, N, K, G, out_dtype):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = fn(to_dev_bf16(X), to_dev_u8(codes), to_dev_f16(scales), N, K, G, out_dtype=out_dtype, d_err=err)
    torch.cuda.synchronize()
    return to_f64(Y), int(err.item())


@pytest.mark.parametrize("M", [3, 16, 40, 64, 100, 300])
@pytest.mark.parametrize("N,K,G", [(300, 1024, 128), (1536, 4096, 64), (9601, 1024, 128), (515, 2048, 256)])
def test_gemm2_tensor_paths(N, K, G, M):
    """The 2-bit codes through the tensor-core kernels: split-K and persistent
    small-M kernels (tq2_gemv and tq2_gemm up to 64 tokens), the prefill
    kernel beyond; sampled token rows compared over every output column."""
    W = synthetic.weights(N, K, index=N + K + G)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    X = synthetic.activations(M, K, offset=1100)
    rows = sorted({0, M // 2, M - 1})
    ref = oracle.linear2(X, codes, scales, N, K, G, rows=rows)
    fns = (tq.gemm2, tq.gemv2) if M <= 64 else (tq.gemm2,)
    for fn in fns:
        Y, e = run_mm2(fn, X, codes, scales, N, K, G, torch.float32)
        assert_rows_close_f32(Y[rows], ref)
        assert e == 0
    Yb, _ = run_mm2(tq.gemm2, X, codes, scales, N, K, G, torch.bfloat16)
    assert_close_bf16(Yb[rows], ref)


@pytest.mark.parametrize("M", [16, 256])
def test_gemm2_rejected_groups(M):
    """Code 3 and bad scales on the tensor paths: NaN output columns and the
    oracle's error bits."""
    N, K, G = 9601, 1024, 128
    W = synthetic.weights(N, K, index=13)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    codes[5, 2, 7] |= 0xC0       # code 3
    codes[4000, 7, 31] = 0xFF    # four codes 3 in a group's last byte
    scales[9600, 1] = 0x7C00     # Inf scale, last row
    scales[130, 0] = 0x8000      # -0 scale
    scales[7777, 3] = 0          # zero group: finite
    X = synthetic.activations(M, K, offset=1101)
    rows = [0, M - 1]
    ref = oracle.linear2(X, codes, scales, N, K, G, rows=rows)
    _, e_ref = oracle.unpack2_bf16(codes, scales, N, K, G)
    Y, e = run_mm2(tq.gemm2, X, codes, scales, N, K, G, torch.float32)
    assert_rows_close_f32(Y[rows], ref)
    assert np.all(np.isnan(Y[:, [5, 4000, 9600, 130]])) and np.all(np.isfinite(Y[:, 7777]))
    assert e == e_ref == tq.DERR_BYTE | tq.DERR_SCALE
