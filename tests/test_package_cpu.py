"""Package files (per-tensor codes + fp16 scales, manifest with hashes, replay).

"precisit/pack-unpack-run", screen.py and test_codec.py descriptions: per-
tensor NPZ files with codes and fp16 scales; the decoder accepts only the
package and checks it; file replay; altering any valid code byte alters the
decoded weights.  Codes come from the oracle; decoding on the CPU side of
these tests is the oracle's.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synthetic
from ternary_weight_only_group_b200 import package as pkg


def make_tensors():
    t = {}
    for i, (name, (N, K), G, fmt) in enumerate([("layers.0.mlp.gate_proj", (48, 256), 64, "base3"),
                                               ("layers.0.mlp.down_proj", (32, 384), 128, "base3"),
                                               ("layers.1/mlp:up proj", (20, 130), 10, "base3"),
                                               ("layers.1.mlp.gate_proj", (24, 256), 64, "2bit"),
                                               ("layers.1.mlp.down_proj", (16, 120), 6, "2bit")]):
        W = synthetic.weights(N, K, index=300 + i)
        c, s, e = (oracle.quantize_pack if fmt == "base3" else oracle.quantize_pack2)(W, G)
        assert e == 0
        t[name] = {"codes": c, "scales": s, "N": N, "K": K, "G": G, "fmt": fmt}
    return t


def decode_cpu(entry):
    f = oracle.unpack_bf16 if entry["fmt"] == "base3" else oracle.unpack2_bf16
    return f(entry["codes"], entry["scales"], entry["N"], entry["K"], entry["G"])


def test_round_trip_bit_exact(tmp_path):
    tensors = make_tensors()
    man = pkg.write_package(str(tmp_path / "p"), tensors)
    back = pkg.read_package(str(tmp_path / "p"))
    assert sorted(back) == sorted(tensors) == sorted(man["tensors"])
    for name, t in tensors.items():
        b = back[name]
        assert np.array_equal(b["codes"], t["codes"]) and np.array_equal(b["scales"], t["scales"])
        assert (b["N"], b["K"], b["G"], b["fmt"]) == (t["N"], t["K"], t["G"], t["fmt"])
        assert np.array_equal(decode_cpu(b)[0], decode_cpu(t)[0])


def test_payload_rates_in_manifest(tmp_path):
    """The page's rates for base-3 (G=64: 1.875 bits per weight, G=128:
    1.75); the 2-bit format stores 8 * (G/4 + 2) / G."""
    man = pkg.write_package(str(tmp_path / "p"), make_tensors())["tensors"]
    assert man["layers.0.mlp.gate_proj"]["payload_bits_per_weight"] == 1.875
    assert man["layers.0.mlp.down_proj"]["payload_bits_per_weight"] == 1.75
    assert man["layers.1.mlp.gate_proj"]["payload_bits_per_weight"] == 2.25


def test_replay_is_byte_identical(tmp_path):
    """Writing the same tensors twice gives the same files (fixed zip
    timestamps and member order), so a package replays to its own hashes."""
    a = pkg.write_package(str(tmp_path / "a"), make_tensors())
    b = pkg.write_package(str(tmp_path / "b"), make_tensors())
    assert a == b
    for e in a["tensors"].values():
        assert open(tmp_path / "a" / e["file"], "rb").read() == open(tmp_path / "b" / e["file"], "rb").read()


def test_damaged_file_rejected(tmp_path):
    d = str(tmp_path / "p")
    man = pkg.write_package(d, make_tensors())
    e = man["tensors"]["layers.0.mlp.down_proj"]
    path = os.path.join(d, e["file"])
    raw = bytearray(open(path, "rb").read())
    raw[-200] ^= 0x01  # a byte near the end of the file
    open(path, "wb").write(bytes(raw))
    with pytest.raises(pkg.PackageError, match="hash"):
        pkg.read_package(d)


def test_changed_code_byte_changes_reconstruction(tmp_path):
    """A valid code byte changed (and the manifest rewritten to match) must
    change the decoded weights."""
    tensors = make_tensors()
    t = tensors["layers.0.mlp.gate_proj"]
    ref = decode_cpu(t)[0]
    c = t["codes"].copy()
    c[3, 1, 5] = (int(c[3, 1, 5]) + 1) % 243
    tensors["layers.0.mlp.gate_proj"] = dict(t, codes=c)
    d = str(tmp_path / "p")
    pkg.write_package(d, tensors)
    got = decode_cpu(pkg.read_package(d)["layers.0.mlp.gate_proj"])[0]
    assert not np.array_equal(got, ref)
    assert np.array_equal(np.delete(got, 3, axis=0), np.delete(ref, 3, axis=0))  # only row 3 changed


def test_missing_extra_and_foreign_files_rejected(tmp_path):
    d = str(tmp_path / "p")
    man = pkg.write_package(d, make_tensors())
    open(os.path.join(d, "stray.npz"), "wb").write(b"x")
    with pytest.raises(pkg.PackageError, match="not in the manifest"):
        pkg.read_package(d)
    os.remove(os.path.join(d, "stray.npz"))
    os.remove(os.path.join(d, man["tensors"]["layers.1.mlp.down_proj"]["file"]))
    with pytest.raises(pkg.PackageError, match="missing"):
        pkg.read_package(d)
    with pytest.raises(pkg.PackageError, match="no manifest"):
        pkg.read_package(str(tmp_path / "nothing-here"))


def test_manifest_shape_mismatch_and_format_rejected(tmp_path):
    d = str(tmp_path / "p")
    pkg.write_package(d, make_tensors())
    mpath = os.path.join(d, pkg.MANIFEST)
    man = json.load(open(mpath))
    man["tensors"]["layers.0.mlp.gate_proj"]["G"] = 128  # shapes no longer agree
    json.dump(man, open(mpath, "w"))
    with pytest.raises(pkg.PackageError, match="codes"):
        pkg.read_package(d)
    man["format"] = "something-else"
    json.dump(man, open(mpath, "w"))
    with pytest.raises(pkg.PackageError, match="format"):
        pkg.read_package(d)


def test_write_refuses_bad_input(tmp_path):
    t = make_tensors()["layers.0.mlp.gate_proj"]
    with pytest.raises(pkg.PackageError):
        pkg.write_package(str(tmp_path / "a"), {"x": dict(t, G=48)})
    with pytest.raises(pkg.PackageError):
        pkg.write_package(str(tmp_path / "b"), {"x": dict(t, scales=t["scales"].astype(np.float32))})
    pkg.write_package(str(tmp_path / "c"), {"x": t})
    with pytest.raises(pkg.PackageError, match="not empty"):
        pkg.write_package(str(tmp_path / "c"), {"x": t})
