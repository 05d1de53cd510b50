"""Decoding from a package only: the arrays a checked package holds, decoded
by the library's unpack kernels, equal the oracle's decoding bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.parity import bits_u16
from ternary_weight_only_group_b200 import package as pkg

pytestmark = pytest.mark.gpu


def test_decode_package_matches_oracle(tmp_path):
    tensors = {}
    for i, (name, (N, K), G, fmt) in enumerate([("gate", (3584, 1024), 64, "base3"),
                                               ("down", (1024, 3584), 128, "base3"),
                                               ("gate2", (3584, 1024), 64, "2bit"),
                                               ("odd", (37, 130), 10, "2bit")]):
        W = synthetic.weights(N, K, index=700 + i)
        c, s, _ = (oracle.quantize_pack if fmt == "base3" else oracle.quantize_pack2)(W, G)
        tensors[name] = {"codes": c, "scales": s, "N": N, "K": K, "G": G, "fmt": fmt}
    d = str(tmp_path / "p")
    pkg.write_package(d, tensors)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = pkg.decode_package(d, d_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for name, t in tensors.items():
        f = oracle.unpack_bf16 if t["fmt"] == "base3" else oracle.unpack2_bf16
        ref, _ = f(t["codes"], t["scales"], t["N"], t["K"], t["G"])
        assert np.array_equal(bits_u16(out[name]).reshape(ref.shape), ref), name
