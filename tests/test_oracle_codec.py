"""Pins for the oracle's scale, trit and base-3 codec.

Every expected value here comes from the pages (golden fixtures), from a
closed form, from a brute-force search in exact rational arithmetic, or from
a library conversion -- never from the oracle's own formulas retyped.
Source for the codec: "precisit/pack-unpack-run", the codec.py and
test_codec.py descriptions and the payload-rate paragraph.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ helpers
# Independent of the oracle: values come from torch / numpy conversions and
# exact rationals; rounding is decided by comparing distances exactly.

def frac_bf16(h: int) -> Fraction:
    v = torch.tensor([h], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).item()
    return Fraction(v)


def frac_fp16(h: int) -> Fraction:
    return Fraction(float(np.array([h], dtype=np.uint16).view(np.float16)[0]))


def bf16_bits(x: float) -> int:
    b = torch.tensor([x], dtype=torch.float64).to(torch.float32).to(torch.bfloat16)
    return int(b.view(torch.int16).item()) & 0xFFFF


def nearest_fp16_even(q: Fraction):
    """Nearest non-negative binary16 to q, ties to the even pattern; None if it overflows."""
    if q >= 65520:
        return None
    c = int(np.array([float(q)], dtype=np.float16).view(np.uint16)[0])
    cands = [b for b in (c - 1, c, c + 1) if 0 <= b < 0x7C00]
    best = min(cands, key=lambda b: (abs(frac_fp16(b) - q), b & 1))
    return best


def bpg(G):
    return -(-G // 5)


# ------------------------------------------------------------------ golden

def test_payload_rate_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "payload_rates.txt"))
            if l.strip() and not l.startswith("#")]
    for G, bpw in rows:
        G = int(G)
        N, K = 8, 2 * G
        W = synthetic.weights(N, K, index=7)
        codes, scales, err = oracle.quantize_pack(W, G)
        assert err == 0
        measured = 8.0 * (codes.nbytes + scales.nbytes) / (N * K)
        assert measured == pytest.approx(float(bpw), abs=1e-12)


def test_payload_rate_formula_all_G():
    # The page's closed form 8*(ceil(G/5)+2)/G, measured from the oracle's
    # output sizes for every G up to 256.
    for G in range(1, 257):
        N, K = 2, G
        W = synthetic.weights(N, K, index=G)
        codes, scales, _ = oracle.quantize_pack(W, G)
        assert codes.shape == (N, 1, math.ceil(G / 5))
        assert 8.0 * (codes.nbytes + scales.nbytes) / (N * K) == pytest.approx(
            8 * (math.ceil(G / 5) + 2) / G, rel=0, abs=1e-12)


def test_ffn_scope_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "ffn_scope.txt"))
            if l.strip() and not l.startswith("#")]
    nmat, nsel, _total = map(int, rows[0])
    layers = nmat // 3
    total = layers * sum(n * k for n, k in synthetic.FFN_SHAPES.values())
    assert nmat == 72 and total == nsel == 264241152


# ------------------------------------------------------------------ codewords

def test_all_243_codewords_against_scalar_base3():
    """All 243 codewords vs the scalar definition sum(d_i * 3^i), d = t + 1,
    first weight = least significant digit; inverse by repeated divmod."""
    one, mone = bf16_bits(1.0), bf16_bits(-1.0)
    seen = set()
    for trits in itertools.product((-1, 0, 1), repeat=5):
        w = np.array([{1: one, -1: mone, 0: 0}[t] for t in trits], dtype=np.uint16)[None, :]
        codes, scales, err = oracle.quantize_pack(w, 5)
        assert err == 0
        byte = int(codes[0, 0, 0])
        expect = sum((t + 1) * 3 ** i for i, t in enumerate(trits))
        assert byte == expect
        seen.add(byte)
        # inverse: digits by repeated divmod
        b, digits = byte, []
        for _ in range(5):
            b, d = divmod(b, 3)
            digits.append(d - 1)
        assert tuple(digits) == trits
    assert seen == set(range(243))


def test_decode_every_valid_byte():
    s = 0x3C00  # binary16 1.0 -> decoded magnitude bf16 1.0
    for b in range(243):
        codes = np.array([[[b]]], dtype=np.uint8)
        out, err = oracle.unpack_bf16(codes, np.array([[s]], dtype=np.uint16), 1, 5, 5)
        assert err == 0
        v, digits = b, []
        for _ in range(5):
            v, d = divmod(v, 3)
            digits.append(d - 1)
        expect = [{1: 0x3F80, -1: 0xBF80, 0: 0}[t] for t in digits]
        assert list(out[0]) == expect


@pytest.mark.parametrize("b", range(243, 256))
def test_invalid_bytes_rejected(b):
    G = 10
    codes = np.full((1, 2, 2), 121, dtype=np.uint8)
    codes[0, 1, 1] = b
    scales = np.array([[0x3C00, 0x3C00]], dtype=np.uint16)
    out, err = oracle.unpack_bf16(codes, scales, 1, 2 * G, G)
    assert err & oracle.ERR_BYTE
    assert np.all(out[0, G:] == 0x7FC0)       # rejected group decodes to NaN
    assert np.all(out[0, :G] == 0)            # the other group is untouched


def test_changed_valid_byte_changes_reconstruction():
    """The page's test list: altering any valid code byte alters the decoded
    weights.  Full bytes: the 243 decodings are pairwise distinct.
    Partial last byte (G=64: 4 digits + 1 padding): any change either
    changes the decoded values or is rejected."""
    scales = np.array([[0x3C00]], dtype=np.uint16)
    outs = set()
    for b in range(243):
        out, err = oracle.unpack_bf16(np.array([[[b]]], dtype=np.uint8), scales, 1, 5, 5)
        outs.add(tuple(out[0]))
    assert len(outs) == 243
    G = 64
    base = np.full((1, 1, bpg(G)), 121, dtype=np.uint8)
    ref, _ = oracle.unpack_bf16(base, scales, 1, G, G)
    for b in range(256):
        if b == 121:
            continue
        c = base.copy()
        c[0, 0, -1] = b
        out, err = oracle.unpack_bf16(c, scales, 1, G, G)
        assert err != 0 or not np.array_equal(out, ref)


@pytest.mark.parametrize("G,real", [(64, 4), (128, 3), (6, 1), (7, 2), (9, 4)])
def test_padding_digits(G, real):
    """The last byte holds G mod 5 real digits; the rest are padding (digit 1).
    A padding digit other than 1 is rejected."""
    scales = np.array([[0x3C00]], dtype=np.uint16)
    for b in range(243):
        c = np.full((1, 1, bpg(G)), 121, dtype=np.uint8)
        c[0, 0, -1] = b
        out, err = oracle.unpack_bf16(c, scales, 1, G, G)
        digits = [(b // 3 ** i) % 3 for i in range(5)]
        canonical = all(d == 1 for d in digits[real:])
        assert bool(err & oracle.ERR_PADDING) == (not canonical)
        if canonical:
            assert err == 0


@pytest.mark.parametrize("G", [5, 10, 15])
def test_no_padding_when_G_multiple_of_5(G):
    scales = np.array([[0x3C00]], dtype=np.uint16)
    c = np.zeros((1, 1, bpg(G)), dtype=np.uint8)  # every digit 0 -> all trits -1
    out, err = oracle.unpack_bf16(c, scales, 1, G, G)
    assert err == 0 and np.all(out == 0xBF80)


def test_zero_group_encoding():
    """A scale of zero gives an all-zero group: every byte 1+3+9+27+81 = 121,
    decoded as +0."""
    for G in (1, 3, 5, 64, 128):
        W = np.zeros((2, 2 * G), dtype=np.uint16)
        W[1, :] = 0x8000  # negative zeros
        codes, scales, err = oracle.quantize_pack(W, G)
        assert err == 0 and np.all(scales == 0) and np.all(codes == 121)
        out, err = oracle.unpack_bf16(codes, scales, 2, 2 * G, G)
        assert err == 0 and np.all(out == 0)


def test_zero_scale_forces_zero_group_on_decode():
    codes = np.zeros((1, 1, 13), dtype=np.uint8)  # all trits -1 ...
    out, err = oracle.unpack_bf16(codes, np.zeros((1, 1), np.uint16), 1, 64, 64)
    assert err & oracle.ERR_PADDING  # digit 0 in the padding slot
    codes[0, 0, -1] = 0 + 1 * 81     # digits 0,0,0,0 real, padding 1
    out, err = oracle.unpack_bf16(codes, np.zeros((1, 1), np.uint16), 1, 64, 64)
    assert err == 0 and np.all(out == 0)  # ... but the scale is zero


@pytest.mark.parametrize("s", [0x7C00, 0xFC00, 0x7E00, 0x8000, 0xBC00])
def test_bad_scale_rejected(s):
    codes = np.full((1, 1, 13), 121, dtype=np.uint8)
    out, err = oracle.unpack_bf16(codes, np.array([[s]], np.uint16), 1, 64, 64)
    assert err & oracle.ERR_SCALE and np.all(out == 0x7FC0)


# ------------------------------------------------------------------ scale

def test_scale_constant_magnitude():
    """A group of copies of +-c has mean c: the scale is RNE_binary16(c),
    which numpy's float64 -> float16 conversion gives in one rounding."""
    rng = np.random.default_rng(11)
    mags = rng.integers(0, 0x7F80, size=3000).astype(np.uint16)
    for a in mags:
        c = float(frac_bf16(int(a)))
        for G in (1, 7, 64):
            signs = rng.integers(0, 2, size=G).astype(np.uint16) << 15
            s, err = oracle.group_scale(a | signs)
            if c >= 65520:
                assert err == oracle.ERR_OVERFLOW and s == 0
            else:
                assert err == 0
                assert s == int(np.array([c], np.float16).view(np.uint16)[0])


def _random_groups(seed, count, G, spread):
    rng = np.random.default_rng(seed)
    e0 = rng.integers(100, 140, size=(count, 1))
    e = np.clip(e0 - rng.integers(0, spread + 1, size=(count, G)), 0, 254)
    f = rng.integers(0, 128, size=(count, G))
    sign = rng.integers(0, 2, size=(count, G))
    return ((sign << 15) | (e << 7) | f).astype(np.uint16)


@pytest.mark.parametrize("G,spread", [(1, 0), (2, 3), (5, 20), (64, 8), (64, 60),
                                      (128, 16), (128, 130), (100, 40), (256, 5)])
def test_scale_vs_exact_rational(G, spread):
    """Exact mean as a Fraction, rounded by exact distance comparison."""
    groups = _random_groups(G * 1000 + spread, 150 if G < 200 else 40, G, spread)
    for w in groups:
        mean = sum(abs(frac_bf16(int(h))) for h in w) / G
        expect = nearest_fp16_even(mean)
        s, err = oracle.group_scale(w)
        if expect is None:
            assert err == oracle.ERR_OVERFLOW and s == 0
        else:
            assert err == 0 and s == expect, (w, mean)


def test_scale_ties_to_even():
    one, tiny = bf16_bits(1.0), bf16_bits(2.0 ** -100)
    # mean = 0.5 + 2^-12: halfway between 0.5 (0x3800, even) and 0.5+2^-11 (0x3801)
    w = [one] * 8 + [bf16_bits(2.0 ** -8)] + [0] * 7
    assert oracle.group_scale(w) == (0x3800, 0)
    # a tiny extra magnitude breaks the tie upwards
    assert oracle.group_scale(w[:-1] + [tiny]) == (0x3801, 0)
    # mean = 0.5 + 3*2^-12: halfway between 0x3801 (odd) and 0x3802 (even)
    w3 = [one] * 8 + [bf16_bits(3 * 2.0 ** -8)] + [0] * 7
    assert oracle.group_scale(w3) == (0x3802, 0)


def test_scale_near_ties_with_wide_exponent_spread():
    """Sums that sit one unit of 2^-53 below a binary16 midpoint times G, plus
    magnitudes far below it: the answer depends on every bit of the sum."""
    two = bf16_bits(2.0)
    fill = [bf16_bits(255 * 2.0 ** -(13 + 8 * i)) for i in range(6)]  # = 2^-5 - 2^-53
    base = [two] * 32 + fill                                             # G=64 sum: 64 + 2^-5 - 2^-53
    mid_lo, mid_hi = 0x3C00, 0x3C01   # 1.0 and 1 + 2^-10; midpoint 1 + 2^-11 = (64 + 2^-5)/64
    pad = lambda xs: xs + [0] * (64 - len(xs))
    assert oracle.group_scale(pad(base)) == (mid_lo, 0)
    t = bf16_bits(2.0 ** -59)
    assert oracle.group_scale(pad(base + [t, t])) == (mid_lo, 0)          # still below
    h = bf16_bits(2.0 ** -54)
    assert oracle.group_scale(pad(base + [h, h])) == (mid_lo, 0)          # exact tie -> even
    assert oracle.group_scale(pad(base + [h, h, t])) == (mid_hi, 0)       # above the tie
    sub = 0x0001                                                          # 2^-133
    assert oracle.group_scale(pad(base + [h, h, sub])) == (mid_hi, 0)


def test_scale_zero_and_underflow():
    assert oracle.group_scale([0] * 64) == (0, 0)
    assert oracle.group_scale([bf16_bits(2.0 ** -25)]) == (0, 0)            # tie at half the smallest subnormal
    assert oracle.group_scale([bf16_bits(1.5 * 2.0 ** -25)]) == (1, 0)      # rounds to 2^-24
    assert oracle.group_scale([bf16_bits(2.0 ** -26)] * 2) == (0, 0)
    assert oracle.group_scale([bf16_bits(2.0 ** -24), 0]) == (0, 0)         # mean 2^-25: tie -> 0
    assert oracle.group_scale([bf16_bits(2.0 ** -24), 1]) == (1, 0)         # + 2^-133 -> 2^-24


def test_scale_overflow():
    assert oracle.group_scale([bf16_bits(65280.0)]) == (0x7BF8, 0)
    assert oracle.group_scale([bf16_bits(65280.0), bf16_bits(65536.0)]) == (0x7BFC, 0)
    assert oracle.group_scale([bf16_bits(65536.0)]) == (0, oracle.ERR_OVERFLOW)
    assert oracle.group_scale([bf16_bits(3e38)] * 3) == (0, oracle.ERR_OVERFLOW)


@pytest.mark.parametrize("bad", [0x7F80, 0xFF80, 0x7FC0, 0x7F81])
def test_nonfinite_weight_flagged(bad):
    w = synthetic.weights(1, 64, index=3)
    w[0, 17] = bad
    codes, scales, err = oracle.quantize_pack(w, 64)
    assert err == oracle.ERR_WEIGHT and scales[0, 0] == 0 and np.all(codes == 121)


# ------------------------------------------------------------------ trits

def test_trit_bruteforce_argmin():
    """clamp(RNE(w/s)) equals the argmin over {-1,0,1} of |w/s - t| with
    ties going to the even candidate (0)."""
    rng = np.random.default_rng(3)
    ws = synthetic.random_bf16_bits(4000, seed=4)
    ss = rng.integers(1, 0x7C00, size=4000).astype(np.uint16)
    for w, s in zip(ws, ss):
        q = frac_bf16(int(w)) / frac_fp16(int(s))
        best = min((-1, 0, 1), key=lambda t: (abs(q - t), t != 0))
        assert oracle.trit(int(w), int(s)) == best


def test_trit_ties_and_clamp():
    for s in (0x3C00, 0x0001, 0x3555, 0x7BFF, 0x2E66):
        sv = frac_fp16(s)
        for mult, expect in ((Fraction(1, 2), 0), (1, 1), (Fraction(3, 2), 1), (Fraction(5, 2), 1), (100, 1)):
            x = sv * mult
            xf = float(x)
            b = bf16_bits(xf)
            if frac_bf16(b) != x:
                continue  # not representable in bf16
            assert oracle.trit(b, s) == expect
            assert oracle.trit(b | 0x8000, s) == -expect
    assert oracle.trit(bf16_bits(5.0), 0) == 0


# ------------------------------------------------------------------ whole codec

def test_tiny_workload_invariants():
    W, X, G = synthetic.tiny_case()
    N, K = W.shape
    codes, scales, err = oracle.quantize_pack(W, G)
    assert err == 0
    assert np.all(scales[:4] == 0) and np.all(codes[:4] == 121)
    assert np.all(scales[4:] != 0) and codes.max() < 243
    out, err = oracle.unpack_bf16(codes, scales, N, K, G)
    assert err == 0
    # every decoded value is +0 or +-RNE_bf16(scale of its group)
    s_bf16 = torch.from_numpy(scales.view(np.float16).astype(np.float32)).to(torch.bfloat16)
    s_bits = s_bf16.view(torch.int16).numpy().view(np.uint16)
    mag = np.repeat(s_bits, G, axis=1)
    o = out
    assert np.all((o == 0) | (o == mag) | (o == (mag | 0x8000)))
    # the sign of a nonzero decoded value is the sign of the weight
    nz = o != 0
    assert np.all((o[nz] >> 15) == (W[nz] >> 15))


def test_requantize_is_idempotent_on_trits():
    """Quantizing decoded weights reproduces the same trits: each nonzero
    decoded magnitude is >= the new group mean, so it is > half of it."""
    W = synthetic.weights(64, 640, index=9, outlier_frac=1e-2)
    for G in (64, 128, 5):
        codes, scales, _ = oracle.quantize_pack(W, G)
        Wd, _ = oracle.unpack_bf16(codes, scales, 64, 640, G)
        codes2, scales2, err = oracle.quantize_pack(Wd, G)
        assert err == 0 and np.array_equal(codes2, codes)
