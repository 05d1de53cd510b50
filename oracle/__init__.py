"""CPU oracle for the ternary weight-only grouped linear layer.

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the CPU
baseline leg of ``bench.py`` may import this module; the product library and
its Python binding never do.  The arithmetic lives in ``tq_oracle.c`` (plain C,
exact integer scale, binary64 matmul); this file only compiles it with gcc and
marshals numpy arrays.  Nothing here shares code with the CUDA path.

Every function cites the passage it follows inside ``tq_oracle.c``.  Pins that
tie it to the pages and to mathematics (not to itself) are in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libtq_oracle.so")
_lock = threading.Lock()
_lib = None

ERR_BYTE = 1
ERR_PADDING = 2
ERR_WEIGHT = 4
ERR_SCALE = 8
ERR_OVERFLOW = 16

MAX_G = 1 << 16


def build(force: bool = False) -> str:
    """Compile tq_oracle.c into oracle/_build/libtq_oracle.so (plain gcc)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u16p = ctypes.POINTER(ctypes.c_uint16)
            u8p = ctypes.POINTER(ctypes.c_uint8)
            i64p = ctypes.POINTER(ctypes.c_int64)
            f64p = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_value.restype = ctypes.c_double
            lib.oracle_fp16_value.argtypes = [ctypes.c_uint16]
            lib.oracle_fp16_value.restype = ctypes.c_double
            lib.oracle_bf16_round.argtypes = [ctypes.c_double]
            lib.oracle_bf16_round.restype = ctypes.c_uint16
            lib.oracle_group_scale.argtypes = [u16p, i64, u16p]
            lib.oracle_group_scale.restype = ctypes.c_uint32
            lib.oracle_trit.argtypes = [ctypes.c_uint16, ctypes.c_uint16]
            lib.oracle_trit.restype = ctypes.c_int
            lib.oracle_bytes_per_group.argtypes = [i64]
            lib.oracle_bytes_per_group.restype = i64
            lib.oracle_quantize_pack.argtypes = [u16p, i64, i64, i64, u8p, u16p]
            lib.oracle_quantize_pack.restype = ctypes.c_uint32
            lib.oracle_unpack_bf16.argtypes = [u8p, u16p, i64, i64, i64, u16p]
            lib.oracle_unpack_bf16.restype = ctypes.c_uint32
            lib.oracle_bytes_per_group2.argtypes = [i64]
            lib.oracle_bytes_per_group2.restype = i64
            lib.oracle_quantize_pack2.argtypes = [u16p, i64, i64, i64, u8p, u16p]
            lib.oracle_quantize_pack2.restype = ctypes.c_uint32
            lib.oracle_unpack2_bf16.argtypes = [u8p, u16p, i64, i64, i64, u16p]
            lib.oracle_unpack2_bf16.restype = ctypes.c_uint32
            u32p = ctypes.POINTER(ctypes.c_uint32)
            lib.oracle_w4_dequant.argtypes = [u32p, u16p, u16p, i64, i64, i64, f64p]
            lib.oracle_w4_dequant.restype = None
            lib.oracle_matmul.argtypes = [u16p, i64, i64p, i64, u16p, i64, i64, f64p]
            lib.oracle_matmul.restype = None
            lib.oracle_matmul_points.argtypes = [u16p, u16p, i64, i64p, i64p, i64, f64p]
            lib.oracle_matmul_points.restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bit patterns, got {a.dtype}")
    return a


def _check_shape(N: int, K: int, G: int):
    if G < 1 or G > MAX_G:
        raise ValueError(f"G={G} out of range [1, {MAX_G}]")
    if N < 0 or K < 0 or K % G:
        raise ValueError(f"K={K} must be a non-negative multiple of G={G}")


# ---------------------------------------------------------------- scalars

def bf16_value(h: int) -> float:
    return _load().oracle_bf16_value(int(h))


def fp16_value(h: int) -> float:
    return _load().oracle_fp16_value(int(h))


def bf16_round(v: float) -> int:
    return int(_load().oracle_bf16_round(float(v)))


def bytes_per_group(G: int) -> int:
    """ceil(G/5): five base-3 digits per byte, each group byte-aligned."""
    return int(_load().oracle_bytes_per_group(int(G)))


def group_scale(w_bits) -> tuple[int, int]:
    """(binary16 scale bits, error bits) of one group of bf16 bit patterns."""
    w = _u16(np.asarray(w_bits, dtype=np.uint16))
    s = ctypes.c_uint16(0)
    err = _load().oracle_group_scale(_ptr(w, ctypes.c_uint16), w.size, ctypes.byref(s))
    return int(s.value), int(err)


def trit(w_bits: int, s_bits: int) -> int:
    """clamp(round_half_even(w / s), -1, 1); 0 when s == 0."""
    return int(_load().oracle_trit(int(w_bits), int(s_bits)))


# ---------------------------------------------------------------- codec

def quantize_pack(W_bits: np.ndarray, G: int):
    """[N, K] bf16 bit patterns -> (codes u8 [N, K/G, ceil(G/5)], scales u16 [N, K/G], err)."""
    W = _u16(W_bits)
    N, K = W.shape
    _check_shape(N, K, G)
    ng, B = K // G, bytes_per_group(G)
    codes = np.zeros((N, ng, B), dtype=np.uint8)
    scales = np.zeros((N, ng), dtype=np.uint16)
    err = _load().oracle_quantize_pack(_ptr(W, ctypes.c_uint16), N, K, G,
                                       _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint16))
    return codes, scales, int(err)


def unpack_bf16(codes: np.ndarray, scales: np.ndarray, N: int, K: int, G: int):
    """codes + scales -> (decoded bf16 bit patterns [N, K], err)."""
    _check_shape(N, K, G)
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = _u16(scales)
    assert c.size == N * (K // G) * bytes_per_group(G) and s.size == N * (K // G)
    out = np.zeros((N, K), dtype=np.uint16)
    err = _load().oracle_unpack_bf16(_ptr(c, ctypes.c_uint8), _ptr(s, ctypes.c_uint16), N, K, G,
                                     _ptr(out, ctypes.c_uint16))
    return out, int(err)


# ---------------------------------------------------------------- 2-bit codec

def bytes_per_group2(G: int) -> int:
    """ceil(G/4): four 2-bit codes per byte, each group byte-aligned."""
    return int(_load().oracle_bytes_per_group2(int(G)))


def quantize_pack2(W_bits: np.ndarray, G: int):
    """[N, K] bf16 bit patterns -> (codes u8 [N, K/G, ceil(G/4)], scales u16 [N, K/G], err),
    2-bit format (code t + 1, first weight in the low bits)."""
    W = _u16(W_bits)
    N, K = W.shape
    _check_shape(N, K, G)
    ng, B = K // G, bytes_per_group2(G)
    codes = np.zeros((N, ng, B), dtype=np.uint8)
    scales = np.zeros((N, ng), dtype=np.uint16)
    err = _load().oracle_quantize_pack2(_ptr(W, ctypes.c_uint16), N, K, G,
                                        _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint16))
    return codes, scales, int(err)


def unpack2_bf16(codes: np.ndarray, scales: np.ndarray, N: int, K: int, G: int):
    """2-bit codes + scales -> (decoded bf16 bit patterns [N, K], err)."""
    _check_shape(N, K, G)
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = _u16(scales)
    assert c.size == N * (K // G) * bytes_per_group2(G) and s.size == N * (K // G)
    out = np.zeros((N, K), dtype=np.uint16)
    err = _load().oracle_unpack2_bf16(_ptr(c, ctypes.c_uint8), _ptr(s, ctypes.c_uint16), N, K, G,
                                      _ptr(out, ctypes.c_uint16))
    return out, int(err)


# ---------------------------------------------------------------- matmul

def matmul(X_bits: np.ndarray, What_bits: np.ndarray, rows=None) -> np.ndarray:
    """Y = X . What^T in binary64 for the selected rows of X (all by default)."""
    X = _u16(X_bits)
    Wd = _u16(What_bits)
    M, K = X.shape
    N, K2 = Wd.shape
    assert K == K2
    if rows is None:
        r = None
        nrows = M
        rp = None
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        assert r.size == 0 or (r.min() >= 0 and r.max() < M)
        nrows = r.size
        rp = _ptr(r, ctypes.c_int64)
    Y = np.zeros((nrows, N), dtype=np.float64)
    _load().oracle_matmul(_ptr(X, ctypes.c_uint16), M, rp, nrows, _ptr(Wd, ctypes.c_uint16), N, K,
                          _ptr(Y, ctypes.c_double))
    return Y


def matmul_points(X_bits: np.ndarray, What_bits: np.ndarray, m_idx, n_idx) -> np.ndarray:
    """Y[i] = sum_k X[m_i, k] * What[n_i, k] in binary64."""
    X = _u16(X_bits)
    Wd = _u16(What_bits)
    K = X.shape[1]
    assert Wd.shape[1] == K
    m = np.ascontiguousarray(m_idx, dtype=np.int64)
    n = np.ascontiguousarray(n_idx, dtype=np.int64)
    assert m.shape == n.shape
    Y = np.zeros(m.shape, dtype=np.float64)
    _load().oracle_matmul_points(_ptr(X, ctypes.c_uint16), _ptr(Wd, ctypes.c_uint16), K,
                                 _ptr(m, ctypes.c_int64), _ptr(n, ctypes.c_int64), m.size,
                                 _ptr(Y, ctypes.c_double))
    return Y


def linear(X_bits, codes, scales, N: int, K: int, G: int, rows=None) -> np.ndarray:
    """The fused layer's definition: Y = X . unpack(codes, scales)^T (binary64)."""
    Wd, _ = unpack_bf16(codes, scales, N, K, G)
    return matmul(X_bits, Wd, rows)


def round_bf16_array(Y: np.ndarray) -> np.ndarray:
    """RNE of binary64 values to bf16 bit patterns (elementwise, via the C helper)."""
    f = _load().oracle_bf16_round
    flat = np.asarray(Y, dtype=np.float64).ravel()
    return np.array([f(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(Y))


def linear2(X_bits, codes, scales, N: int, K: int, G: int, rows=None) -> np.ndarray:
    """The fused layer on the 2-bit format: Y = X . unpack2(codes, scales)^T (binary64)."""
    Wd, _ = unpack2_bf16(codes, scales, N, K, G)
    return matmul(X_bits, Wd, rows)


# ---------------------------------------------------------------- W4A16 affine format

def w4_dequant(codes: np.ndarray, scales: np.ndarray, biases: np.ndarray, N: int, K: int, G: int) -> np.ndarray:
    """codes uint32 [N, K/8] (first code in the low nibble), bf16 scales and
    biases [N, K/G] -> binary64 weights q * s + b [N, K]."""
    if G < 1 or K % G or K % 8:
        raise ValueError(f"K={K} must be a multiple of G={G} and of 8")
    c = np.ascontiguousarray(codes, dtype=np.uint32)
    s = _u16(scales)
    b = _u16(biases)
    assert c.size == N * (K // 8) and s.size == N * (K // G) and b.size == N * (K // G)
    out = np.zeros((N, K), dtype=np.float64)
    _load().oracle_w4_dequant(_ptr(c, ctypes.c_uint32), _ptr(s, ctypes.c_uint16), _ptr(b, ctypes.c_uint16),
                              N, K, G, _ptr(out, ctypes.c_double))
    return out


def linear_w4(X_bits, codes, scales, biases, N: int, K: int, G: int) -> np.ndarray:
    """Y = X . W^T with W the W4 weights reconstructed in binary64 and X bf16
    widened exactly; the products and sums in binary64 (numpy matmul)."""
    X = _u16(X_bits)
    xv = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return xv @ w4_dequant(codes, scales, biases, N, K, G).T
