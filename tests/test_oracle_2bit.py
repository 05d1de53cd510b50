"""Pins for the oracle's 2-bit ternary format (four codes per byte).

Source: "Autoregressive Language Model on the 6502 Processor", summary:
BitNet ternary weights (-1, 0, 1) stored four parameters per byte.  The page
fixes only the density; the code assignment (c = t + 1), the bit order (first
weight in the low bits), byte-aligned groups with padding code 1 and the
rejection of code 3 are readings chosen to mirror the base-3 codec.

Expected values come from the page's density figure, from bytes worked out
by hand from those readings, from brute force over all 256 bytes decoded with
plain integer arithmetic in this file, and from the base-3 oracle (pinned on
its own), which must decode the same weights from the same matrix.
"""
import numpy as np
import pytest

import oracle
import synthetic

BF16_ONE, BF16_MINUS_ONE = 0x3F80, 0xBF80


def test_density_four_per_byte():
    """52k parameters in 13 KB: four per byte whenever G is a multiple of 4."""
    assert 52_000 // 4 == 13_000
    for G in (4, 8, 16, 64, 128, 256):
        N, K = 13, 4000 // G * G
        assert N * (K // G) * oracle.bytes_per_group2(G) * 4 == N * K
    assert [oracle.bytes_per_group2(G) for G in (1, 2, 3, 4, 5, 6, 7, 8, 9)] == [1, 1, 1, 1, 2, 2, 2, 2, 3]


def test_worked_byte():
    """One group of four, worked by hand: W = (1, 0, -1, 1), mean |w| = 0.75
    (binary16 0x3A00); trits (1, 0, -1, 1), codes (2, 1, 0, 2) from the low
    bits up: 2 + 1*4 + 0*16 + 2*64 = 134."""
    W = np.array([[BF16_ONE, 0x0000, BF16_MINUS_ONE, BF16_ONE]], dtype=np.uint16)
    codes, scales, err = oracle.quantize_pack2(W, 4)
    assert err == 0 and scales.tolist() == [[0x3A00]] and codes.tolist() == [[[134]]]
    Wd, e = oracle.unpack2_bf16(codes, scales, 1, 4, 4)
    assert e == 0 and Wd.tolist() == [[0x3F40, 0x0000, 0xBF40, 0x3F40]]  # +-0.75 in bf16


def test_worked_padding():
    """G = 6: two bytes per group; weights 6 and 7 are padding (code 1).
    W = (-1, -1, 1, 1, 0, 1): mean 5/6, trits (-1, -1, 1, 1, 0, 1).
    Byte 0 = codes (0, 0, 2, 2) = 0 + 0 + 32 + 128 = 160;
    byte 1 = codes (1, 2, pad 1, pad 1) = 1 + 8 + 16 + 64 = 89."""
    W = np.array([[BF16_MINUS_ONE, BF16_MINUS_ONE, BF16_ONE, BF16_ONE, 0x0000, BF16_ONE]], dtype=np.uint16)
    codes, scales, err = oracle.quantize_pack2(W, 6)
    assert err == 0 and codes.tolist() == [[[160, 89]]]
    # a padding code other than 1 is rejected (error bit 2), the group decodes
    # to NaN: code 0 at weight 6 (89 - 16) or code 2 at weight 7 (89 + 64)
    for bad in (73, 153):
        c = codes.copy()
        c[0, 0, 1] = bad
        Wd, e = oracle.unpack2_bf16(c, scales, 1, 6, 6)
        assert e == oracle.ERR_PADDING and np.all(Wd == 0x7FC0)


def test_decode_every_byte_bruteforce():
    """All 256 bytes as one group of four with scale 1.0 (binary16 0x3C00):
    a byte holding a code 3 is rejected (error bit 1, NaN group); otherwise
    weight i is (((b >> 2i) & 3) - 1) * 1.0."""
    for b in range(256):
        c = np.array([[[b]]], dtype=np.uint8)
        Wd, e = oracle.unpack2_bf16(c, np.array([[0x3C00]], dtype=np.uint16), 1, 4, 4)
        fields = [(b >> (2 * i)) & 3 for i in range(4)]
        if 3 in fields:
            assert e == oracle.ERR_BYTE and np.all(Wd == 0x7FC0)
        else:
            want = [{0: BF16_MINUS_ONE, 1: 0x0000, 2: BF16_ONE}[f] for f in fields]
            assert e == 0 and Wd.tolist() == [want], b


@pytest.mark.parametrize("G", [4, 6, 8, 16, 64, 128, 130])
def test_same_weights_as_base3(G):
    """Scale and trits are those of the base-3 codec: decoding either format
    gives the same bf16 weights, bit for bit, including zero groups, tiny and
    huge groups and non-finite weights (both flag them and store zero groups)."""
    N, K = 5, 4 * G
    W = synthetic.weights(N, K, index=G)
    W[0, :G] = 0                       # all-zero group
    W[1, G:2 * G] = 0x0001             # subnormal magnitudes
    W[2, 0] = 0x7F80                   # +Inf weight: flagged, zero group
    W[3, 3 * G - 1] = 0x7F7F           # largest finite bf16: the mean overflows binary16
    c3, s3, e3 = oracle.quantize_pack(W, G)
    c2, s2, e2 = oracle.quantize_pack2(W, G)
    assert e2 == e3 and np.array_equal(s2, s3)
    W3, f3 = oracle.unpack_bf16(c3, s3, N, K, G)
    W2, f2 = oracle.unpack2_bf16(c2, s2, N, K, G)
    assert f2 == f3 == 0 and np.array_equal(W2, W3)
    assert c2.shape == (N, K // G, (G + 3) // 4)


def test_bad_scales_rejected():
    for s in (0x7C00, 0xFC00, 0x7E00, 0x8000, 0x8001):
        c = np.full((1, 1, 4), 0x55, dtype=np.uint8)  # codes 1: zero trits
        Wd, e = oracle.unpack2_bf16(c, np.array([[s]], dtype=np.uint16), 1, 16, 16)
        assert e == oracle.ERR_SCALE and np.all(Wd == 0x7FC0)


def test_linear2_small_bruteforce():
    """Y = X . What^T for a 3 x 20 by 4 x 20 case, summed here in binary64
    from values widened by numpy (every product of two bf16 values is exact
    in binary64, and at these magnitudes so are the short sums)."""
    G, N, K, M = 4, 4, 20, 3
    W = synthetic.weights(N, K, index=7)
    X = synthetic.activations(M, K)
    codes, scales, _ = oracle.quantize_pack2(W, G)
    Y = oracle.linear2(X, codes, scales, N, K, G)
    Wd, _ = oracle.unpack2_bf16(codes, scales, N, K, G)
    xf = X.astype(np.uint32) << 16
    wf = Wd.astype(np.uint32) << 16
    xv = xf.view(np.float32).astype(np.float64)
    wv = wf.view(np.float32).astype(np.float64)
    for m in range(M):
        for n in range(N):
            assert Y[m, n] == sum(xv[m, k] * wv[n, k] for k in range(K))
