"""Package files for packed ternary weights.

"precisit/pack-unpack-run", screen.py and test_codec.py descriptions: the
packer writes per-tensor NPZ files holding the codes and the fp16 scales; the
decoder accepts only the package and checks it; a packed file must replay to
the same reconstruction.  This module is host-side IO: it writes and checks
packages, and `decode_package` hands their arrays to the library's unpack
kernels (there is no CPU decoder here).

Layout of a package directory:
  manifest.json   {"format": "tq-package-1", "tensors": {name: entry}}, where
                  entry = {"file", "sha256", "bytes", "N", "K", "G", "fmt",
                  "payload_bits_per_weight"}; fmt is "base3" (five digits per
                  byte) or "2bit" (four codes per byte)
  <file>.npz      arrays "codes" (uint8 [N, K/G, B]) and "scales" (uint16
                  binary16 bit patterns [N, K/G]), stored uncompressed with
                  fixed zip timestamps so that equal tensors give equal bytes
A reader rejects a package whose manifest names a missing file, whose file
hash or array shapes disagree with the manifest, or whose directory holds
files the manifest does not name.  Like the format on that page, this is not
a loader for untrusted third-party packages: the checks catch damage and
mix-ups, not an adversary who rewrites the manifest too.
"""
from __future__ import annotations

import hashlib
import io
import json
import os
import re
import zipfile

import numpy as np

FORMAT = "tq-package-1"
MANIFEST = "manifest.json"
FORMATS = ("base3", "2bit")
_ZIP_TIME = (1980, 1, 1, 0, 0, 0)


class PackageError(ValueError):
    """A package that is damaged, incomplete or inconsistent with its manifest."""


def bytes_per_group_fmt(G: int, fmt: str) -> int:
    if fmt == "base3":
        return (G + 4) // 5
    if fmt == "2bit":
        return (G + 3) // 4
    raise PackageError(f"unknown format {fmt!r}")


def payload_bits_per_weight(G: int, fmt: str) -> float:
    """8 * (bytes per group + 2) / G: codes, padding and the binary16 scale."""
    return 8.0 * (bytes_per_group_fmt(G, fmt) + 2) / G


def _sha256(path: str) -> str:
    h = hashlib.sha256()
    with open(path, "rb") as f:
        for chunk in iter(lambda: f.read(1 << 20), b""):
            h.update(chunk)
    return h.hexdigest()


def _file_name(name: str) -> str:
    safe = re.sub(r"[^A-Za-z0-9_.-]", "_", name)
    return f"{safe}-{hashlib.sha256(name.encode()).hexdigest()[:8]}.npz"


def _write_npz(path: str, arrays: dict):
    """An .npz (zip of .npy members) with fixed member order and timestamps."""
    with zipfile.ZipFile(path, "w", compression=zipfile.ZIP_STORED) as z:
        for key in sorted(arrays):
            buf = io.BytesIO()
            np.lib.format.write_array(buf, np.ascontiguousarray(arrays[key]), allow_pickle=False)
            info = zipfile.ZipInfo(f"{key}.npy", date_time=_ZIP_TIME)
            info.external_attr = 0o644 << 16
            z.writestr(info, buf.getvalue())


def _as_u16(scales) -> np.ndarray:
    a = np.ascontiguousarray(scales)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    if a.dtype != np.uint16:
        raise PackageError(f"scales must be float16 or uint16 bit patterns, got {a.dtype}")
    return a


def _check_arrays(name, codes, scales, N, K, G, fmt):
    if G < 1 or K < 0 or N < 0 or K % G:
        raise PackageError(f"{name}: bad shape N={N} K={K} G={G}")
    want_c = (N, K // G, bytes_per_group_fmt(G, fmt))
    if codes.dtype != np.uint8 or tuple(codes.shape) != want_c:
        raise PackageError(f"{name}: codes {codes.dtype}{tuple(codes.shape)}, expected uint8{want_c}")
    if scales.dtype != np.uint16 or tuple(scales.shape) != (N, K // G):
        raise PackageError(f"{name}: scales {scales.dtype}{tuple(scales.shape)}, expected uint16{(N, K // G)}")


def write_package(directory: str, tensors: dict, extra: dict | None = None) -> dict:
    """Write `tensors` (name -> dict(codes, scales, N, K, G, fmt)) into a new
    or empty directory; returns the manifest."""
    os.makedirs(directory, exist_ok=True)
    if os.listdir(directory):
        raise PackageError(f"{directory} is not empty")
    entries = {}
    for name in sorted(tensors):
        t = tensors[name]
        fmt = t.get("fmt", "base3")
        N, K, G = int(t["N"]), int(t["K"]), int(t["G"])
        if G < 1 or K < 0 or N < 0 or K % G:
            raise PackageError(f"{name}: bad shape N={N} K={K} G={G}")
        try:
            codes = np.ascontiguousarray(t["codes"], dtype=np.uint8).reshape(
                N, K // G, bytes_per_group_fmt(G, fmt))
            scales = _as_u16(t["scales"]).reshape(N, K // G)
        except ValueError as ex:
            raise PackageError(f"{name}: arrays do not match N={N} K={K} G={G} {fmt}: {ex}") from None
        _check_arrays(name, codes, scales, N, K, G, fmt)
        fname = _file_name(name)
        path = os.path.join(directory, fname)
        _write_npz(path, {"codes": codes, "scales": scales})
        entries[name] = {"file": fname, "sha256": _sha256(path), "bytes": os.path.getsize(path),
                         "N": N, "K": K, "G": G, "fmt": fmt,
                         "payload_bits_per_weight": payload_bits_per_weight(G, fmt)}
    manifest = {"format": FORMAT, "tensors": entries, "extra": extra or {}}
    with open(os.path.join(directory, MANIFEST), "w") as f:
        json.dump(manifest, f, indent=1, sort_keys=True)
        f.write("\n")
    return manifest


def read_manifest(directory: str) -> dict:
    path = os.path.join(directory, MANIFEST)
    if not os.path.isfile(path):
        raise PackageError(f"{directory}: no {MANIFEST}")
    with open(path) as f:
        manifest = json.load(f)
    if manifest.get("format") != FORMAT:
        raise PackageError(f"{directory}: format {manifest.get('format')!r}, expected {FORMAT!r}")
    return manifest


def read_package(directory: str) -> dict:
    """Check the package and return name -> dict(codes, scales, N, K, G, fmt)
    with scales as uint16 bit patterns.  Raises PackageError on any mismatch."""
    manifest = read_manifest(directory)
    entries = manifest["tensors"]
    listed = {e["file"] for e in entries.values()}
    present = set(os.listdir(directory)) - {MANIFEST}
    if present - listed:
        raise PackageError(f"{directory}: files not in the manifest: {sorted(present - listed)}")
    out = {}
    for name in sorted(entries):
        e = entries[name]
        path = os.path.join(directory, e["file"])
        if not os.path.isfile(path):
            raise PackageError(f"{name}: {e['file']} is missing")
        if os.path.getsize(path) != e["bytes"] or _sha256(path) != e["sha256"]:
            raise PackageError(f"{name}: {e['file']} does not match its manifest hash")
        with np.load(path, allow_pickle=False) as z:
            if sorted(z.files) != ["codes", "scales"]:
                raise PackageError(f"{name}: members {sorted(z.files)}")
            codes, scales = z["codes"], z["scales"]
        N, K, G, fmt = int(e["N"]), int(e["K"]), int(e["G"]), e["fmt"]
        _check_arrays(name, codes, scales, N, K, G, fmt)
        out[name] = {"codes": codes, "scales": scales, "N": N, "K": K, "G": G, "fmt": fmt}
    return out


def decode_package(directory: str, device="cuda", d_err=None) -> dict:
    """Check the package, then decode every tensor to bf16 [N, K] on `device`
    with the library's unpack kernels (tq_unpack_bf16 / tq2_unpack_bf16)."""
    import torch

    import ternary_weight_only_group_b200 as tq
    out = {}
    for name, t in read_package(directory).items():
        codes = torch.from_numpy(t["codes"]).to(device)
        scales = torch.from_numpy(t["scales"].view(np.float16)).to(device)
        unpack = tq.unpack_bf16 if t["fmt"] == "base3" else tq.unpack2_bf16
        out[name] = unpack(codes, scales, t["N"], t["K"], t["G"], d_err=d_err)
    return out
