"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host before touching CUDA (runs without a GPU)."""
import ctypes
import os
import re

import pytest

import ternary_weight_only_group_b200 as tq
from ternary_weight_only_group_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    return tq.lib()


def header_symbols():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    return sorted(set(re.findall(r"TQ_API\s+[\w\s\*]*?\b(tq2?_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    syms = header_symbols()
    assert syms == sorted(tq.EXPORTS)
    L = tq.lib()
    for s in syms:
        assert hasattr(L, s), s


def test_version_and_status_strings():
    assert "sm_100a" in tq.version()
    for st, name in enumerate(["TQ_OK", "TQ_ERR_INVALID_ARG", "TQ_ERR_ALIGNMENT",
                               "TQ_ERR_UNSUPPORTED", "TQ_ERR_CUDA"]):
        assert tq.status_string(st) == name


@pytest.mark.parametrize("N,K,G", [(256, 640, 64), (3584, 1024, 128), (1024, 3584, 64),
                                   (3, 15, 5), (1, 1, 1), (0, 128, 64), (7, 4096, 4096)])
def test_size_queries(N, K, G):
    assert tq.codes_bytes(N, K, G) == N * (K // G) * -(-G // 5)
    assert tq.scales_bytes(N, K, G) == N * (K // G) * 2
    assert tq.workspace_bytes(1, N, K, G) >= 0
    assert tq.codes2_bytes(N, K, G) == N * (K // G) * -(-G // 4)


@pytest.mark.parametrize("N,K,G", [(4, 100, 64), (4, 64, 0), (4, 64, -1), (-1, 64, 64),
                                   (4, -64, 64), (4, 8192, 8192)])
def test_size_queries_reject_bad_shapes(N, K, G):
    assert tq.codes_bytes(N, K, G) == 0 and tq.scales_bytes(N, K, G) == 0
    assert tq.codes2_bytes(N, K, G) == 0


def fake(addr):
    return ctypes.c_void_p(addr)


# Host-side validation: every call below must fail before any CUDA call.
BAD_CALLS = [
    ("G=0", lambda L: L.tq_quantize_pack(fake(0x1000), 4, 64, 0, fake(0x9000), fake(0xA000), None, None),
     tq.TQ_ERR_INVALID_ARG),
    ("K%G", lambda L: L.tq_quantize_pack(fake(0x1000), 4, 100, 64, fake(0x9000), fake(0xA000), None, None),
     tq.TQ_ERR_INVALID_ARG),
    ("G>max", lambda L: L.tq_quantize_pack(fake(0x1000), 1, 8192, 8192, fake(0x90000), fake(0xA0000), None, None),
     tq.TQ_ERR_INVALID_ARG),
    ("null W", lambda L: L.tq_quantize_pack(None, 4, 64, 64, fake(0x9000), fake(0xA000), None, None),
     tq.TQ_ERR_INVALID_ARG),
    ("null codes", lambda L: L.tq_quantize_pack(fake(0x1000), 4, 64, 64, None, fake(0xA000), None, None),
     tq.TQ_ERR_INVALID_ARG),
    ("overlap", lambda L: L.tq_quantize_pack(fake(0x1000), 4, 64, 64, fake(0x1010), fake(0xA000), None, None),
     tq.TQ_ERR_INVALID_ARG),
    ("W misaligned", lambda L: L.tq_quantize_pack(fake(0x1008), 4, 64, 64, fake(0x9000), fake(0xA000), None, None),
     tq.TQ_ERR_ALIGNMENT),
    ("scales odd", lambda L: L.tq_quantize_pack(fake(0x1000), 4, 64, 64, fake(0x9000), fake(0xA001), None, None),
     tq.TQ_ERR_ALIGNMENT),
    ("unpack out misaligned", lambda L: L.tq_unpack_bf16(fake(0x9000), fake(0xA000), 4, 64, 64, fake(0x1002), None, None),
     tq.TQ_ERR_ALIGNMENT),
    ("unpack overlap", lambda L: L.tq_unpack_bf16(fake(0x1000), fake(0xA000), 4, 64, 64, fake(0x1000), None, None),
     tq.TQ_ERR_INVALID_ARG),
    ("gemv bad dtype", lambda L: L.tq_gemv(fake(0x1000), 1, fake(0x9000), fake(0xA000), 4, 64, 64, fake(0xB000), 7,
                                           None, 0, None, None), tq.TQ_ERR_INVALID_ARG),
    ("gemv M<0", lambda L: L.tq_gemv(fake(0x1000), -1, fake(0x9000), fake(0xA000), 4, 64, 64, fake(0xB000), 0,
                                     None, 0, None, None), tq.TQ_ERR_INVALID_ARG),
    ("gemv Y aliases X", lambda L: L.tq_gemv(fake(0x1000), 2, fake(0x9000), fake(0xA000), 4, 64, 64, fake(0x1040),
                                             0, None, 0, None, None), tq.TQ_ERR_INVALID_ARG),
    ("gemv X misaligned", lambda L: L.tq_gemv(fake(0x1004), 1, fake(0x9000), fake(0xA000), 4, 64, 64, fake(0xB000),
                                              0, None, 0, None, None), tq.TQ_ERR_ALIGNMENT),
    ("gemv Y f32 misaligned", lambda L: L.tq_gemv(fake(0x1000), 1, fake(0x9000), fake(0xA000), 4, 64, 64,
                                                  fake(0xB002), 0, None, 0, None, None), tq.TQ_ERR_ALIGNMENT),
    ("gemm null scales", lambda L: L.tq_gemm(fake(0x1000), 1, fake(0x9000), None, 4, 64, 64, fake(0xB000), 1,
                                             None, 0, None, None), tq.TQ_ERR_INVALID_ARG),
    ("gemm K%G", lambda L: L.tq_gemm(fake(0x1000), 1, fake(0x9000), fake(0xA000), 4, 96, 64, fake(0xB000), 1,
                                     None, 0, None, None), tq.TQ_ERR_INVALID_ARG),
    ("2-bit pack G=0", lambda L: L.tq2_quantize_pack(fake(0x1000), 4, 64, 0, fake(0x9000), fake(0xA000), None,
                                                     None), tq.TQ_ERR_INVALID_ARG),
    ("2-bit pack codes misaligned", lambda L: L.tq2_quantize_pack(fake(0x1000), 4, 64, 64, fake(0x9002),
                                                                  fake(0xA000), None, None), tq.TQ_ERR_ALIGNMENT),
    ("2-bit pack overlap", lambda L: L.tq2_quantize_pack(fake(0x1000), 4, 64, 64, fake(0x1100), fake(0xA000),
                                                         None, None), tq.TQ_ERR_INVALID_ARG),
    ("2-bit unpack codes misaligned", lambda L: L.tq2_unpack_bf16(fake(0x9001), fake(0xA000), 4, 64, 64,
                                                                  fake(0x1000), None, None), tq.TQ_ERR_ALIGNMENT),
    ("2-bit unpack null scales", lambda L: L.tq2_unpack_bf16(fake(0x9000), None, 4, 64, 64, fake(0x1000), None,
                                                             None), tq.TQ_ERR_INVALID_ARG),
    ("2-bit gemv codes misaligned", lambda L: L.tq2_gemv(fake(0x1000), 1, fake(0x9002), fake(0xA000), 4, 64, 64,
                                                         fake(0xB000), 0, None, 0, None, None), tq.TQ_ERR_ALIGNMENT),
    ("2-bit gemv Y overlaps codes", lambda L: L.tq2_gemv(fake(0x1000), 1, fake(0x9000), fake(0xA000), 4, 64, 64,
                                                         fake(0x9010), 0, None, 0, None, None), tq.TQ_ERR_INVALID_ARG),
    ("2-bit gemv K%G", lambda L: L.tq2_gemv(fake(0x1000), 1, fake(0x9000), fake(0xA000), 4, 96, 64,
                                            fake(0xB000), 0, None, 0, None, None), tq.TQ_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("name,call,expect", BAD_CALLS, ids=[c[0] for c in BAD_CALLS])
def test_host_validation(name, call, expect):
    assert call(tq.lib()) == expect


def test_empty_inputs_are_noops():
    L = tq.lib()
    assert L.tq_quantize_pack(None, 0, 64, 64, None, None, None, None) == tq.TQ_OK
    assert L.tq_unpack_bf16(None, None, 0, 128, 64, None, None, None) == tq.TQ_OK
    assert L.tq_gemv(None, 0, fake(0x9000), fake(0xA000), 4, 64, 64, None, 0, None, 0, None, None) == tq.TQ_OK
    assert L.tq2_quantize_pack(None, 0, 64, 64, None, None, None, None) == tq.TQ_OK
    assert L.tq2_unpack_bf16(None, None, 0, 128, 64, None, None, None) == tq.TQ_OK
    assert L.tq2_gemv(None, 0, fake(0x9000), fake(0xA000), 4, 64, 64, None, 0, None, 0, None, None) == tq.TQ_OK


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    monkeypatch.setattr(tq, "_lib", None)
    monkeypatch.setattr(tq, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        tq.lib()
