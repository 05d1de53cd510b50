"""Comparison helpers for the GPU parity tests (test code only)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances stated for the fused matmul outputs:
#   fp32 output: max_n |gpu - oracle| <= 1e-3 * max_n |oracle| on every output row;
#   bf16 output: |gpu - oracle| <= 2e-2 + 2e-2 * |oracle| elementwise.
F32_ROW_REL = 1e-3
BF16_RTOL = 2e-2
BF16_ATOL = 2e-2


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_dev_u8(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)


def to_dev_f16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.float16)).to(device)


def bits_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def assert_rows_close_f32(gpu: np.ndarray, ref: np.ndarray, rel: float = F32_ROW_REL):
    """Per output row: identical NaN positions; max|gpu-ref| <= rel * max|ref|."""
    gpu = np.atleast_2d(gpu)
    ref = np.atleast_2d(ref)
    assert gpu.shape == ref.shape
    nan_g, nan_r = np.isnan(gpu), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"NaN mismatch at {np.argwhere(nan_g != nan_r)[:5]}"
    g = np.where(nan_r, 0.0, gpu)
    r = np.where(nan_r, 0.0, ref)
    err = np.max(np.abs(g - r), axis=1)
    bound = rel * np.max(np.abs(r), axis=1)
    bad = err > bound
    assert not bad.any(), (f"rows {np.nonzero(bad)[0][:5]}: err {err[bad][:5]} > bound {bound[bad][:5]}")


def assert_close_bf16(gpu: np.ndarray, ref: np.ndarray, rtol=BF16_RTOL, atol=BF16_ATOL):
    nan_g, nan_r = np.isnan(gpu), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r)
    g = np.where(nan_r, 0.0, gpu)
    r = np.where(nan_r, 0.0, ref)
    bad = np.abs(g - r) > atol + rtol * np.abs(r)
    assert not bad.any(), f"{bad.sum()} elements out of tolerance, first {np.argwhere(bad)[:5]}"
