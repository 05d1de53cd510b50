"""The bounded waits of the tensor-core kernels give up cleanly.

Every mbarrier wait of the three tcgen05 kernels (split-K small-M, persistent
small-M, prefill) is bounded; when a wait runs out the kernel sets
TQ_DERR_TIMEOUT, stops issuing work, lets its copies and MMAs in flight land,
frees its tensor memory and returns.  To make a wait run out without faulting
anything, the library's test hook withholds the first activation load of
every CTA (TQ_DEBUG_WITHHOLD_X_LOAD=1: the mbarrier it would complete is never
completed) with a short bound (TQ_DEBUG_WAIT_LIMIT_NS).  The test checks the
error bit, that the call returns within a bounded time, and that the next
ordinary call on the same stream -- which allocates tensor memory on the same
SMs again -- reproduces the reference output bit for bit.
"""
import os
import time

import numpy as np
import pytest
import torch

import oracle
import synthetic
import ternary_weight_only_group_b200 as tq
from tests.parity import assert_rows_close_f32, to_dev_bf16, to_dev_f16, to_dev_u8, to_f64

pytestmark = pytest.mark.gpu

# (route, function, M, N, K, G): the kernel each shape reaches
ROUTES = [("split-K small-M", tq.gemv, 16, 300, 1024, 128),
          ("persistent small-M", tq.gemv, 16, 9600, 1024, 128),
          ("prefill", tq.gemm, 256, 512, 1024, 128)]


def call(fn, X, codes, scales, N, K, G):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = torch.full((X.shape[0], N), 7.0, dtype=torch.float32, device="cuda")
    fn(X, codes, scales, N, K, G, out=Y, d_err=err)
    torch.cuda.synchronize()
    return to_f64(Y), int(err.item())


@pytest.mark.parametrize("route,fn,M,N,K,G", ROUTES, ids=[r[0] for r in ROUTES])
def test_wait_gives_up_and_next_call_is_exact(route, fn, M, N, K, G):
    W = synthetic.weights(N, K, index=61 + N)
    codes_h, scales_h, _ = oracle.quantize_pack(W, G)
    X_h = synthetic.activations(M, K, offset=900)
    rows = [0, M // 2, M - 1]
    ref = oracle.linear(X_h, codes_h, scales_h, N, K, G, rows=rows)
    X, codes, scales = to_dev_bf16(X_h), to_dev_u8(codes_h), to_dev_f16(scales_h)

    Y0, e0 = call(fn, X, codes, scales, N, K, G)
    assert e0 == 0
    assert_rows_close_f32(Y0[rows], ref)

    os.environ["TQ_DEBUG_WAIT_LIMIT_NS"] = str(20_000_000)  # 20 ms
    os.environ["TQ_DEBUG_WITHHOLD_X_LOAD"] = "1"
    try:
        t0 = time.perf_counter()
        _, e1 = call(fn, X, codes, scales, N, K, G)
        elapsed = time.perf_counter() - t0
    finally:
        del os.environ["TQ_DEBUG_WAIT_LIMIT_NS"]
        del os.environ["TQ_DEBUG_WITHHOLD_X_LOAD"]
    assert e1 & tq.DERR_TIMEOUT, f"{route}: no timeout bit ({e1})"
    assert elapsed < 5.0, f"{route}: the aborted call took {elapsed:.2f} s"

    for _ in range(2):  # tensor memory was released: the same SMs allocate it again
        Y2, e2 = call(fn, X, codes, scales, N, K, G)
        assert e2 == 0
        assert np.array_equal(Y2, Y0), f"{route}: the call after the timeout differs"
