"""GPU parity of decode matmuls chained the way a decode step runs them.

Every launch of tq_gemv / tq2_gemv is a programmatic dependent of the kernel
before it on the stream: it reads its codes and scales before waiting for
that kernel and its activations only after.  Here a chain of layers is
captured in one CUDA graph with real data dependencies -- layer l's bf16
output buffer IS layer l+1's input -- and replayed; each layer's output is
compared with the oracle:

  * per layer, on the input the GPU actually consumed (the previous GPU
    layer's output): the single-launch tolerance of the matmul
    (|gpu - oracle| <= 2e-2 + 2e-2 |oracle| for bf16 outputs);
  * along the pure oracle chain (oracle matmul, RNE to bf16, fed forward):
    the same rtol = atol = 2e-2 on every layer.

The weights are drawn with sigma = 1 / sqrt(0.44 K) (the decoded ternary
layer then roughly preserves the activations' unit variance), so that the
absolute tolerance stays small against the values at every depth.

The ordering rule of include/tq.h is exercised in both directions: a
quantize call directly followed by a matmul on the same code buffers (the
quantizer never releases its dependents early and makes its stores visible
before its blocks exit), and a matmul directly followed by a quantize call
that overwrites the buffers the matmul reads.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import assert_close_bf16, bits_u16, to_dev_bf16, to_dev_f16, to_dev_u8

pytestmark = pytest.mark.gpu

LAYERS = 8
# (name, [(N, K) per hop]); the hops alternate so that each output feeds the next input
CHAINS = {
    # 0.8 MB layers: the pre-decode kernel (weights decoded before the wait), M <= 8
    "ffn": [(3584, 1024), (1024, 3584)],
    # matrices whose rows do not fit the pre-decode kernel: lookup tables at
    # M <= 2, the tensor-core small-M kernels at M >= 3
    "large": [(16384, 1024), (1024, 16384)],
}


@functools.lru_cache(maxsize=8)
def chain_weights(name, G, fmt):
    """Oracle-packed weights for LAYERS layers (the hops repeat)."""
    hop_shapes = CHAINS[name.rstrip("2")]
    packs = []
    for l in range(LAYERS):
        N, K = hop_shapes[l % len(hop_shapes)]
        W = synthetic.weights(N, K, index=4000 + 17 * l + G + (len(name) << 8),
                              sigma=float(1.0 / np.sqrt(0.44 * K)))
        if fmt == 3:
            codes, scales, _ = oracle.quantize_pack(W, G)
        else:
            codes, scales, _ = oracle.quantize_pack2(W, G)
        packs.append((N, K, codes, scales))
    return packs


def oracle_layer(X_bits, pack, G, fmt):
    N, K, codes, scales = pack
    if fmt == 3:
        return oracle.linear(X_bits, codes, scales, N, K, G)
    return oracle.linear2(X_bits, codes, scales, N, K, G)


def run_chain_graph(packs, X0_bits, G, fmt, replays=2):
    """Capture the chain in one graph (Y_l is X_{l+1}), replay it; returns the
    bf16 bit patterns of every layer's output from each replay."""
    M = X0_bits.shape[0]
    fn = tq.gemv if fmt == 3 else tq.gemv2
    dev = [(N, K, to_dev_u8(c), to_dev_f16(s)) for (N, K, c, s) in packs]
    X0 = to_dev_bf16(X0_bits)
    Ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for (N, _, _, _) in dev]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        x = X0
        for (N, K, c, s), y in zip(dev, Ys):
            fn(x, c, s, N, K, G, out=y, d_err=err)
            x = y

    step()  # once outside capture (kernel attributes)
    torch.cuda.synchronize()
    for y in Ys:
        y.fill_(float("nan"))
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="relaxed"):
        step()
    outs = []
    for _ in range(replays):
        for y in Ys:
            y.fill_(float("nan"))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        outs.append([bits_u16(y) for y in Ys])
    assert int(err.item()) == 0
    del graph
    return outs


def check_chain(packs, X0_bits, G, fmt):
    outs = run_chain_graph(packs, X0_bits, G, fmt)
    # replays are deterministic
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b), "graph replays differ"
    gpu = outs[0]
    x_gpu = X0_bits
    x_ref = X0_bits
    for l, pack in enumerate(packs):
        y_gpu = synthetic_bits_to_f64(gpu[l])
        # (1) this launch on the input it consumed
        ref_here = oracle_layer(x_gpu, pack, G, fmt)
        assert_close_bf16(y_gpu, ref_here)
        # (2) the pure oracle chain
        ref_chain = oracle_layer(x_ref, pack, G, fmt)
        assert_close_bf16(y_gpu, ref_chain)
        assert np.std(ref_chain) > 0.2, "activations collapsed: the comparison would be vacuous"
        x_gpu = gpu[l]
        x_ref = oracle.round_bf16_array(ref_chain)


def synthetic_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("M", [1, 2, 8])
def test_ffn_chain_predecode(G, M):
    packs = chain_weights("ffn", G, 3)
    X0 = synthetic.activations(M, packs[0][1], offset=600)
    check_chain(packs, X0, G, 3)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_large_chain(G, M):
    packs = chain_weights("large", G, 3)
    X0 = synthetic.activations(M, packs[0][1], offset=601)
    check_chain(packs, X0, G, 3)


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("M", [1, 3])
def test_ffn_chain_2bit(G, M):
    packs = chain_weights("ffn2", G, 2)
    X0 = synthetic.activations(M, packs[0][1], offset=602)
    check_chain(packs, X0, G, 2)


@pytest.mark.parametrize("fmt", [3, 2])
@pytest.mark.parametrize("N,K,G", [(3584, 1024, 64), (16384, 1024, 128)])
def test_quantize_then_gemv_same_stream(fmt, N, K, G):
    """quantize_pack into the very buffers the next launch reads, alternating
    two weight matrices in one graph: every gemv must see the codes written
    by the quantize call just before it, never the previous matrix's."""
    sig = float(1.0 / np.sqrt(0.44 * K))
    Wa = synthetic.weights(N, K, index=4500 + fmt, sigma=sig)
    Wb = synthetic.weights(N, K, index=4600 + fmt, sigma=sig)
    X = synthetic.activations(1, K, offset=603)
    if fmt == 3:
        ref = [oracle.linear(X, *oracle.quantize_pack(W, G)[:2], N, K, G) for W in (Wa, Wb)]
        qp, mm = tq.quantize_pack, tq.gemv
    else:
        ref = [oracle.linear2(X, *oracle.quantize_pack2(W, G)[:2], N, K, G) for W in (Wa, Wb)]
        qp, mm = tq.quantize_pack2, tq.gemv2
    dW = [to_dev_bf16(Wa), to_dev_bf16(Wb)]
    dX = to_dev_bf16(X)
    codes, scales = qp(dW[1], G)  # start from the other matrix's codes
    Ys = [torch.empty((1, N), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def quantize_into(W):
        f = tq.lib().tq_quantize_pack if fmt == 3 else tq.lib().tq2_quantize_pack
        rc = f(W.data_ptr(), N, K, G, codes.data_ptr(), scales.data_ptr(), err.data_ptr(),
               torch.cuda.current_stream().cuda_stream)
        assert rc == tq.TQ_OK

    def step():
        for i in range(4):
            quantize_into(dW[i % 2])
            mm(dX, codes, scales, N, K, G, out=Ys[i], d_err=err)

    step()
    torch.cuda.synchronize()
    for i in range(4):
        assert_close_bf16(synthetic_bits_to_f64(bits_u16(Ys[i])), ref[i % 2])
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="relaxed"):
        step()
    for _ in range(3):
        for y in Ys:
            y.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for i in range(4):
            assert_close_bf16(synthetic_bits_to_f64(bits_u16(Ys[i])), ref[i % 2])
    assert int(err.item()) == 0
    del graph
