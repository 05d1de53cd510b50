"""GPU parity of tq_quantize_pack and tq_unpack_bf16 against the oracle.

Bit-exact on scales, code bytes, decoded bf16 weights and error bits.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import bits_u16, to_dev_bf16, to_dev_f16, to_dev_u8

pytestmark = pytest.mark.gpu


def bf16_bits(x: float) -> int:
    return int(torch.tensor([x], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF


def gpu_pack(W_bits, G):
    W = to_dev_bf16(W_bits)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = tq.quantize_pack(W, G, d_err=err)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), bits_u16(scales), int(err.item())


def gpu_unpack(codes, scales_bits, N, K, G):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tq.unpack_bf16(to_dev_u8(codes), to_dev_f16(scales_bits), N, K, G, d_err=err)
    torch.cuda.synchronize()
    return bits_u16(out), int(err.item())


def check_pack(W_bits, G):
    c_ref, s_ref, e_ref = oracle.quantize_pack(W_bits, G)
    c, s, e = gpu_pack(W_bits, G)
    assert np.array_equal(s.reshape(s_ref.shape), s_ref), np.argwhere(s.reshape(s_ref.shape) != s_ref)[:8]
    assert np.array_equal(c.reshape(c_ref.shape), c_ref), np.argwhere(c.reshape(c_ref.shape) != c_ref)[:8]
    assert e == e_ref
    return c_ref, s_ref


def check_unpack(codes, scales, N, K, G):
    w_ref, e_ref = oracle.unpack_bf16(codes, scales, N, K, G)
    w, e = gpu_unpack(codes, scales, N, K, G)
    assert np.array_equal(w.reshape(w_ref.shape), w_ref), np.argwhere(w.reshape(w_ref.shape) != w_ref)[:8]
    assert e == e_ref


def test_tiny_workload():
    W, X, G = synthetic.tiny_case()
    codes, scales = check_pack(W, G)
    assert np.all(scales[:4] == 0)
    check_unpack(codes, scales, W.shape[0], W.shape[1], G)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("name", ["gate", "down"])
def test_ffn_full_size(name, G):
    W = synthetic.ffn_matrix(name)
    codes, scales = check_pack(W, G)
    check_unpack(codes, scales, W.shape[0], W.shape[1], G)


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 7, 8, 16, 24, 32, 40, 100, 256, 320, 4096])
def test_group_sizes(G):
    K = G * max(2, 512 // G)
    N = 37  # ragged against the groups-per-warp of every fast path
    W = synthetic.weights(N, K, index=G, outlier_frac=0.01)
    W[5] = synthetic.random_bf16_bits(K, seed=G)        # every exponent
    W[6] = 0
    W[7, : K // 2] = 0x0001                               # subnormals only in the first half
    codes, scales = check_pack(W, G)
    check_unpack(codes, scales, N, K, G)


def constructed_groups_64():
    """Groups of 64 whose scale needs every bit of the exact sum, plus edge cases."""
    two = bf16_bits(2.0)
    fill = [bf16_bits(255 * 2.0 ** -(13 + 8 * i)) for i in range(6)]  # sums to 2^-5 - 2^-53
    base = [two] * 32 + fill
    t, h, sub = bf16_bits(2.0 ** -59), bf16_bits(2.0 ** -54), 0x0001
    one = bf16_bits(1.0)
    rows = [
        base, base + [t, t], base + [h, h], base + [h, h, t], base + [h, h, sub],
        [one] * 8 + [bf16_bits(2.0 ** -8)],                  # exact tie -> even
        [one] * 8 + [bf16_bits(2.0 ** -8), bf16_bits(2.0 ** -100)],
        [one] * 8 + [bf16_bits(3 * 2.0 ** -8)],
        [bf16_bits(2.0 ** -19)],                             # mean 2^-25: tie -> 0
        [bf16_bits(2.0 ** -19), 1],                          # just above -> 2^-24
        [bf16_bits(65280.0)] * 64,
        [bf16_bits(65536.0)] * 64,                           # overflow
        [bf16_bits(3e38)],                                   # overflow, huge
        [0x7F80], [0xFFC1], [0x0001] * 64, [0x8000] * 64,
        [bf16_bits(1e-30), bf16_bits(-1.0)],                 # wide spread, slow path
    ]
    W = np.zeros((len(rows), 64), dtype=np.uint16)
    for i, r in enumerate(rows):
        W[i, : len(r)] = r
    rng = np.random.default_rng(1)
    W = W[:, rng.permutation(64)]                            # positions must not matter
    return W


@pytest.mark.parametrize("G", [64, 128, 32])
def test_constructed_edge_groups(G):
    W64 = constructed_groups_64()
    W = W64.reshape(-1, G) if G <= 64 else np.concatenate([W64, np.zeros_like(W64)], axis=1)
    check_pack(W, G)


def test_signs_of_mean_ties_in_trits():
    # |w| == s/2 exactly -> 0 ; |w| == s -> +-1 (G=8: six values of 1.0, two of 0.5 -> mean 0.875)
    W = np.array([[bf16_bits(v) for v in (1.0, 1.0, -1.0, 1.0, 1.0, 1.0, 0.4375, -0.4375)]], dtype=np.uint16)
    codes, scales = check_pack(W, 8)


def test_unpack_every_codeword_fast_path():
    G = 64
    B = 13
    N = 243
    codes = np.empty((N, 1, B), dtype=np.uint8)
    for b in range(243):
        codes[b, 0, :12] = b
        codes[b, 0, 12] = (b % 81) + 81  # last byte: 4 real digits from b, padding digit 1
    scales = np.full((N, 1), 0x2E66, dtype=np.uint16)
    check_unpack(codes, scales, N, G, G)


@pytest.mark.parametrize("G", [64, 128, 40, 5])
def test_unpack_rejections(G):
    N, K = 50, 4 * G
    W = synthetic.weights(N, K, index=3)
    codes, scales, _ = oracle.quantize_pack(W, G)
    rng = np.random.default_rng(G)
    B = codes.shape[2]
    for n in range(0, N, 3):
        g = rng.integers(0, K // G)
        kind = n % 4
        if kind == 0:
            codes[n, g, rng.integers(0, B)] = rng.integers(243, 256)
        elif kind == 1 and G % 5:
            real = G - 5 * (B - 1)
            codes[n, g, B - 1] = (codes[n, g, B - 1] % 3 ** real) + 0 * 3 ** real  # padding digit 0
        elif kind == 2:
            scales[n, g] = [0x7C00, 0xFC00, 0x7E01, 0x8001][n % 4]
        else:
            scales[n, g] = 0  # zero group
    check_unpack(codes, scales, N, K, G)


def test_stacked_gate_up_sampled_rows():
    """The 24-layer gate/up stack as one [172032 x 1024] matrix (the bulk
    workload's first launch) packed on the GPU; sampled rows vs the oracle."""
    N, K, G = 48 * 3584, 1024, 128
    W = np.concatenate([synthetic.ffn_matrix(n, layer=l, outliers=False)
                        for l in range(24) for n in ("gate", "up")])
    c, s, e = gpu_pack(W, G)
    assert e == 0
    rows = np.random.default_rng(0).choice(N, size=256, replace=False)
    c_ref, s_ref, _ = oracle.quantize_pack(W[rows], G)
    assert np.array_equal(c.reshape(N, K // G, -1)[rows], c_ref)
    assert np.array_equal(s.reshape(N, K // G)[rows], s_ref)
    w, e = gpu_unpack(c, s, N, K, G)
    w_ref, _ = oracle.unpack_bf16(c_ref, s_ref, len(rows), K, G)
    assert e == 0 and np.array_equal(w.reshape(N, K)[rows], w_ref)
