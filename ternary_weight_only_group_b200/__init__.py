"""Python binding of libtq, the B200 ternary weight-only grouped linear layer.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libtq.so`` (built in-tree for sm_100a by ``_build.py``).  PyTorch
supplies device memory and the current CUDA stream.  If the library is not
built, importing the functions below raises; there is no CPU fallback.

The raw C entry points are exposed under their C names (``tq_quantize_pack``,
``tq_unpack_bf16``, ``tq_gemv``, ``tq_gemm``, ...) through ``lib()``; the
tensor-level helpers ``quantize_pack``, ``unpack_bf16``, ``gemv`` and ``gemm``
call them with ``tensor.data_ptr()`` and raise ``TQError`` on a non-OK status.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_ALIGNMENT, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA = range(5)
TQ_OUT_F32, TQ_OUT_BF16 = 0, 1
DERR_BYTE, DERR_PADDING, DERR_WEIGHT, DERR_SCALE, DERR_OVERFLOW, DERR_TIMEOUT = 1, 2, 4, 8, 16, 32
MAX_G = 4096

EXPORTS = ("tq_codes_bytes", "tq_scales_bytes", "tq_workspace_bytes", "tq_quantize_pack",
           "tq_unpack_bf16", "tq_gemv", "tq_gemm", "tq2_codes_bytes", "tq2_quantize_pack",
           "tq2_unpack_bf16", "tq2_gemv", "tq2_gemm", "tq_w4_codes_bytes", "tq_w4_gemv", "tq_w4_gemm", "tq_status_string",
           "tq_version")

_lock = threading.Lock()
_lib = None


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load libtq.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   f"`python {os.path.join(HERE, '_build.py')}` (needs nvcc)")
            L = ctypes.CDLL(LIB_PATH)
            i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
            L.tq_codes_bytes.argtypes = [i64, i64, i32]
            L.tq_codes_bytes.restype = sz
            L.tq_scales_bytes.argtypes = [i64, i64, i32]
            L.tq_scales_bytes.restype = sz
            L.tq_workspace_bytes.argtypes = [i64, i64, i64, i32]
            L.tq_workspace_bytes.restype = sz
            L.tq_quantize_pack.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp]
            L.tq_quantize_pack.restype = i32
            L.tq_unpack_bf16.argtypes = [vp, vp, i64, i64, i32, vp, vp, vp]
            L.tq_unpack_bf16.restype = i32
            mm = [vp, i64, vp, vp, i64, i64, i32, vp, i32, vp, sz, vp, vp]
            L.tq_gemv.argtypes = mm
            L.tq_gemv.restype = i32
            L.tq_gemm.argtypes = mm
            L.tq_gemm.restype = i32
            L.tq2_codes_bytes.argtypes = [i64, i64, i32]
            L.tq2_codes_bytes.restype = sz
            L.tq2_quantize_pack.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp]
            L.tq2_quantize_pack.restype = i32
            L.tq2_unpack_bf16.argtypes = [vp, vp, i64, i64, i32, vp, vp, vp]
            L.tq2_unpack_bf16.restype = i32
            L.tq2_gemv.argtypes = mm
            L.tq2_gemv.restype = i32
            L.tq2_gemm.argtypes = mm
            L.tq2_gemm.restype = i32
            L.tq_w4_codes_bytes.argtypes = [i64, i64, i32]
            L.tq_w4_codes_bytes.restype = sz
            L.tq_w4_gemv.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, vp, i32, vp]
            L.tq_w4_gemv.restype = i32
            L.tq_w4_gemm.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, vp, i32, vp]
            L.tq_w4_gemm.restype = i32
            L.tq_status_string.argtypes = [i32]
            L.tq_status_string.restype = ctypes.c_char_p
            L.tq_version.argtypes = []
            L.tq_version.restype = ctypes.c_char_p
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().tq_status_string(int(status)).decode()


def version() -> str:
    return lib().tq_version().decode()


def codes_bytes(N: int, K: int, G: int) -> int:
    return int(lib().tq_codes_bytes(N, K, G))


def scales_bytes(N: int, K: int, G: int) -> int:
    return int(lib().tq_scales_bytes(N, K, G))


def workspace_bytes(M: int, N: int, K: int, G: int) -> int:
    return int(lib().tq_workspace_bytes(M, N, K, G))


def bytes_per_group(G: int) -> int:
    return (G + 4) // 5


def codes2_bytes(N: int, K: int, G: int) -> int:
    return int(lib().tq2_codes_bytes(N, K, G))


def bytes_per_group2(G: int) -> int:
    return (G + 3) // 4


# ----------------------------------------------------------------------------
# tensor-level helpers (torch tensors on the current CUDA device)

def _torch():
    import torch
    return torch


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(status: int, where: str):
    if status != TQ_OK:
        raise TQError(status, where)


def _as_cuda(t, dtype, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def quantize_pack(W, G: int, d_err=None, stream=None):
    """W: [N, K] bf16 CUDA tensor -> (codes uint8 [N, K/G, ceil(G/5)], scales fp16 [N, K/G])."""
    torch = _torch()
    W = _as_cuda(W, torch.bfloat16, "W")
    N, K = W.shape
    if G < 1 or K % G:
        raise TQError(TQ_ERR_INVALID_ARG, "quantize_pack")
    codes = torch.empty((N, K // G, bytes_per_group(G)), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, K // G), dtype=torch.float16, device=W.device)
    _check(lib().tq_quantize_pack(_ptr(W), N, K, G, _ptr(codes), _ptr(scales), _ptr(d_err),
                                  _stream(stream)), "tq_quantize_pack")
    return codes, scales


def unpack_bf16(codes, scales, N: int, K: int, G: int, out=None, d_err=None, stream=None):
    """codes + scales -> [N, K] bf16 decoded weights."""
    torch = _torch()
    codes = _as_cuda(codes, torch.uint8, "codes")
    scales = _as_cuda(scales, torch.float16, "scales")
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=codes.device)
    _check(lib().tq_unpack_bf16(_ptr(codes), _ptr(scales), N, K, G, _ptr(out), _ptr(d_err),
                                _stream(stream)), "tq_unpack_bf16")
    return out


def _matmul(fn, name, X, codes, scales, N, K, G, out_dtype, out, d_err, stream, workspace):
    torch = _torch()
    X = _as_cuda(X, torch.bfloat16, "X")
    codes = _as_cuda(codes, torch.uint8, "codes")
    scales = _as_cuda(scales, torch.float16, "scales")
    M = X.shape[0]
    if X.dim() != 2 or X.shape[1] != K:
        raise ValueError("X must be [M, K]")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=X.device)
    yt = TQ_OUT_BF16 if out.dtype == torch.bfloat16 else TQ_OUT_F32
    ws_need = workspace_bytes(M, N, K, G)
    if workspace is None and ws_need:
        raise ValueError(f"{name} needs {ws_need} bytes of workspace")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(fn(_ptr(X), M, _ptr(codes), _ptr(scales), N, K, G, _ptr(out), yt, _ptr(workspace),
              ws_bytes, _ptr(d_err), _stream(stream)), name)
    return out


def gemv(X, codes, scales, N: int, K: int, G: int, out_dtype=None, out=None, d_err=None,
         stream=None, workspace=None):
    """Decode matmul on the CUDA cores: Y[M, N] = X . What^T (fp32 accumulation)."""
    torch = _torch()
    return _matmul(lib().tq_gemv, "tq_gemv", X, codes, scales, N, K, G,
                   out_dtype or torch.float32, out, d_err, stream, workspace)


def gemm(X, codes, scales, N: int, K: int, G: int, out_dtype=None, out=None, d_err=None,
         stream=None, workspace=None):
    """Prefill matmul on the tensor cores: Y[M, N] = X . What^T (fp32 accumulation)."""
    torch = _torch()
    return _matmul(lib().tq_gemm, "tq_gemm", X, codes, scales, N, K, G,
                   out_dtype or torch.bfloat16, out, d_err, stream, workspace)


# ----------------------------------------------------------------------------
# the 2-bit ternary format (four codes per byte)

def quantize_pack2(W, G: int, d_err=None, stream=None):
    """W: [N, K] bf16 CUDA tensor -> (codes uint8 [N, K/G, ceil(G/4)], scales fp16 [N, K/G])."""
    torch = _torch()
    W = _as_cuda(W, torch.bfloat16, "W")
    N, K = W.shape
    if G < 1 or K % G:
        raise TQError(TQ_ERR_INVALID_ARG, "quantize_pack2")
    codes = torch.empty((N, K // G, bytes_per_group2(G)), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, K // G), dtype=torch.float16, device=W.device)
    _check(lib().tq2_quantize_pack(_ptr(W), N, K, G, _ptr(codes), _ptr(scales), _ptr(d_err),
                                   _stream(stream)), "tq2_quantize_pack")
    return codes, scales


def unpack2_bf16(codes, scales, N: int, K: int, G: int, out=None, d_err=None, stream=None):
    """2-bit codes + scales -> [N, K] bf16 decoded weights."""
    torch = _torch()
    codes = _as_cuda(codes, torch.uint8, "codes")
    scales = _as_cuda(scales, torch.float16, "scales")
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=codes.device)
    _check(lib().tq2_unpack_bf16(_ptr(codes), _ptr(scales), N, K, G, _ptr(out), _ptr(d_err),
                                 _stream(stream)), "tq2_unpack_bf16")
    return out


def gemv2(X, codes, scales, N: int, K: int, G: int, out_dtype=None, out=None, d_err=None,
          stream=None, workspace=None):
    """Decode matmul on the 2-bit format (CUDA cores): Y[M, N] = X . What^T."""
    torch = _torch()
    return _matmul(lib().tq2_gemv, "tq2_gemv", X, codes, scales, N, K, G,
                   out_dtype or torch.float32, out, d_err, stream, workspace)


def gemm2(X, codes, scales, N: int, K: int, G: int, out_dtype=None, out=None, d_err=None,
          stream=None, workspace=None):
    """Prefill matmul on the 2-bit format (tensor cores): Y[M, N] = X . What^T."""
    torch = _torch()
    return _matmul(lib().tq2_gemm, "tq2_gemm", X, codes, scales, N, K, G,
                   out_dtype or torch.bfloat16, out, d_err, stream, workspace)


# ----------------------------------------------------------------------------
# the W4A16 affine format (uint4 codes, bf16 scale and bias per group)

def w4_gemv(X, codes, scales, biases, N: int, K: int, G: int, out_dtype=None, out=None, stream=None):
    """Decode matmul on the W4 format (CUDA cores): Y[M, N] = X . (q * s + b)^T.
    codes: int32/uint32 [N, K/8]; scales, biases: bf16 [N, K/G]."""
    return _w4_matmul(lib().tq_w4_gemv, "tq_w4_gemv", X, codes, scales, biases, N, K, G,
                      out_dtype, out, stream)


def w4_gemm(X, codes, scales, biases, N: int, K: int, G: int, out_dtype=None, out=None, stream=None):
    """Prefill matmul on the W4 format (tensor cores): Y[M, N] = X . (q * s + b)^T."""
    return _w4_matmul(lib().tq_w4_gemm, "tq_w4_gemm", X, codes, scales, biases, N, K, G,
                      out_dtype, out, stream)


def _w4_matmul(fn, name, X, codes, scales, biases, N, K, G, out_dtype, out, stream):
    torch = _torch()
    X = _as_cuda(X, torch.bfloat16, "X")
    if not isinstance(codes, torch.Tensor) or not codes.is_cuda or codes.dtype not in (torch.int32, torch.uint32):
        raise TypeError("codes must be an int32 or uint32 CUDA tensor")
    if not codes.is_contiguous():
        raise ValueError("codes must be contiguous")
    scales = _as_cuda(scales, torch.bfloat16, "scales")
    biases = _as_cuda(biases, torch.bfloat16, "biases")
    M = X.shape[0]
    if X.dim() != 2 or X.shape[1] != K:
        raise ValueError("X must be [M, K]")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.float32, device=X.device)
    yt = TQ_OUT_BF16 if out.dtype == torch.bfloat16 else TQ_OUT_F32
    _check(fn(_ptr(X), M, _ptr(codes), _ptr(scales), _ptr(biases), N, K, G, _ptr(out), yt,
              _stream(stream)), name)
    return out
