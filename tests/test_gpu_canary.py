"""Red-zone canaries around every output buffer.

compute-sanitizer is not available on this machine, so out-of-bounds writes are
caught the plain way: each output (codes, scales, decoded weights, Y) is a
slice in the middle of a larger allocation whose 256-byte red zones on both
sides hold a byte pattern, and the pattern must be intact after the call.
The shapes reach every kernel of each entry point, with ragged row counts.
"""
import numpy as np
import pytest
import torch

import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import to_dev_bf16

pytestmark = pytest.mark.gpu

RED = 256
PATTERN = 0xA5


class Guarded:
    """A uint8 device buffer of `nbytes` with red zones; .view(dtype, shape)."""

    def __init__(self, nbytes, align=256):
        self.raw = torch.full((nbytes + 2 * RED + align,), PATTERN, dtype=torch.uint8, device="cuda")
        base = self.raw.data_ptr()
        self.off = RED + (-(base + RED)) % align
        self.nbytes = nbytes

    def view(self, dtype, shape):
        t = self.raw[self.off:self.off + self.nbytes].view(dtype)
        return t.view(shape)

    def intact(self):
        torch.cuda.synchronize()
        h = self.raw.cpu().numpy()
        return bool(np.all(h[:self.off] == PATTERN) and np.all(h[self.off + self.nbytes:] == PATTERN))


def weights_dev(N, K, index):
    return to_dev_bf16(synthetic.weights(N, K, index=index, outlier_frac=1e-3))


@pytest.mark.parametrize("fmt", [3, 2])
@pytest.mark.parametrize("N,K,G", [(37, 640, 64), (1031, 1024, 128), (13, 1000, 40), (9, 512, 256), (100, 96, 8),
                                   (3, 4096, 4096), (61, 60, 6)])
def test_codec_outputs(fmt, N, K, G):
    if fmt == 2 and G % 2:
        pytest.skip("2-bit codes need 4-byte aligned rows only through the byte count")
    W = weights_dev(N, K, N + G)
    B = (G + 4) // 5 if fmt == 3 else (G + 3) // 4
    gc = Guarded(N * (K // G) * B)
    gs = Guarded(N * (K // G) * 2)
    codes, scales = gc.view(torch.uint8, (N, K // G, B)), gs.view(torch.float16, (N, K // G))
    f = tq.lib().tq_quantize_pack if fmt == 3 else tq.lib().tq2_quantize_pack
    st = torch.cuda.current_stream().cuda_stream
    assert f(W.data_ptr(), N, K, G, codes.data_ptr(), scales.data_ptr(), None, st) == tq.TQ_OK
    assert gc.intact() and gs.intact()
    gw = Guarded(N * K * 2)
    Wd = gw.view(torch.bfloat16, (N, K))
    (tq.unpack_bf16 if fmt == 3 else tq.unpack2_bf16)(codes, scales, N, K, G, out=Wd)
    assert gw.intact()


# (M, N, K, G): pre-decode, lookup tables, streaming tables, row kernel,
# split-K and persistent small-M kernels, prefill
MATMUL = [(1, 3584, 1024, 64), (2, 20011, 1024, 128), (1, 16391, 1024, 64), (1, 4501, 3584, 128),
          (3, 77, 1000, 40), (16, 300, 1024, 128), (16, 9601, 1024, 128), (100, 515, 1024, 128)]


@pytest.mark.parametrize("M,N,K,G", MATMUL)
@pytest.mark.parametrize("yt", [torch.float32, torch.bfloat16])
def test_matmul_outputs(M, N, K, G, yt):
    W = weights_dev(N, K, 3 * N + K)
    codes, scales = tq.quantize_pack(W, G)
    X = to_dev_bf16(synthetic.activations(M, K, offset=1000))
    esz = 4 if yt == torch.float32 else 2
    gy = Guarded(M * N * esz)
    Y = gy.view(yt, (M, N))
    (tq.gemm if M >= 100 else tq.gemv)(X, codes, scales, N, K, G, out=Y)
    assert gy.intact()
    assert torch.isfinite(Y).all()


@pytest.mark.parametrize("M,N,K,G", [(1, 3585, 1024, 64), (3, 999, 2048, 128), (9, 100, 512, 32)])
def test_gemv2_outputs(M, N, K, G):
    W = weights_dev(N, K, N)
    codes, scales = tq.quantize_pack2(W, G)
    X = to_dev_bf16(synthetic.activations(M, K, offset=1001))
    gy = Guarded(M * N * 4)
    Y = gy.view(torch.float32, (M, N))
    tq.gemv2(X, codes, scales, N, K, G, out=Y)
    assert gy.intact()


@pytest.mark.parametrize("M,N,K,G", [(1, 3585, 1024, 128), (5, 1001, 3584, 64), (2, 77, 1000, 40)])
def test_w4_outputs(M, N, K, G):
    codes, scales, biases = synthetic.w4_params(N, K, G, index=N)
    X = to_dev_bf16(synthetic.activations(M, K, offset=1002))
    gy = Guarded(M * N * 2)
    Y = gy.view(torch.bfloat16, (M, N))
    tq.w4_gemv(X, torch.from_numpy(codes.view(np.int32)).cuda(), to_dev_bf16(scales), to_dev_bf16(biases),
               N, K, G, out=Y)
    assert gy.intact()
