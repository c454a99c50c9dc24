"""Build ``libattn.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m exact_tiled_attention_39_b200.build`` (or call
``build()``).  The library is a plain shared object with a C ABI
(``include/attn.h``); it links the CUDA runtime statically and resolves the
driver's tensor-map encoder at run time, so it needs only the NVIDIA driver
at load time.
"""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libattn.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-v",
]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libattn.so")
    return cand


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh")))


def _deps() -> list[str]:
    return sources() + [os.path.join(ROOT, "include", "attn.h"), __file__]


def source_hash(defines: dict[str, str] | None = None) -> str:
    """SHA-256 over the names and bytes of every file the library is built
    from, the compiler flags and any extra defines."""
    h = hashlib.sha256()
    for path in _deps():
        h.update(os.path.relpath(path, ROOT).encode())
        with open(path, "rb") as f:
            h.update(f.read())
    h.update(repr(NVCC_FLAGS).encode())
    h.update(repr(sorted((defines or {}).items())).encode())
    return h.hexdigest()


def _stamp(lib_path: str) -> str:
    return lib_path + ".src-sha256"


def _current(lib_path: str, digest: str) -> bool:
    """True when lib_path exists and was built from sources with this hash
    (recorded in a stamp file beside it).  File times are not trusted: a
    copied tree can carry a binary newer than its sources."""
    if not os.path.exists(lib_path) or not os.path.exists(_stamp(lib_path)):
        return False
    with open(_stamp(lib_path)) as f:
        return f.read().strip() == digest


def up_to_date() -> bool:
    return _current(LIB, source_hash())


def build(force: bool = False, verbose: bool = False) -> str:
    digest = source_hash()
    if not force and _current(LIB, digest):
        return LIB
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"),
           os.path.join(CSRC, "attn_api.cu"), "-o", LIB + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building libattn.so")
    os.replace(LIB + ".tmp", LIB)
    with open(_stamp(LIB), "w") as f:
        f.write(digest + "\n")
    with open(os.path.join(PKG, "build_ptxas.log"), "w") as f:
        f.write(res.stderr)
    return LIB


def build_variant(name: str, defines: dict[str, str]) -> str:
    """Build ``libattn_<name>.so`` in-tree with extra preprocessor defines
    (test builds: the failure-detection test uses one); rebuilt when the
    source hash differs from the one recorded beside it."""
    out = os.path.join(PKG, f"libattn_{name}.so")
    digest = source_hash(defines)
    if _current(out, digest):
        return out
    cmd = [_nvcc(), *[f for f in NVCC_FLAGS if f not in ("-Xptxas", "-v")],
           *[f"-D{k}={v}" for k, v in defines.items()], "-I", os.path.join(ROOT, "include"),
           os.path.join(CSRC, "attn_api.cu"), "-o", out + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building libattn_{name}.so")
    os.replace(out + ".tmp", out)
    with open(_stamp(out), "w") as f:
        f.write(digest + "\n")
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
