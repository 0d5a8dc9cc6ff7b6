"""Builds libs2attn.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m sparse_attention_attn_b200.build          # build if sources changed
    python -m sparse_attention_attn_b200.build --force  # always rebuild

The library is plain CUDA C++ compiled by nvcc; it links only the CUDA runtime
(statically) and resolves cuTensorMapEncodeTiled through the runtime's driver
entry-point query, so it needs no libcuda at link time.
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
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libs2attn.so")
STAMP = LIB + ".srchash"

SOURCES = ["s2attn.cu", "s2_fwd.cu", "s2_bwd.cu", "s2_bwd_fused.cu", "s2_rope.cu", "s2_segment.cu", "s2_nf4.cu"]
HEADERS = ["s2_ptx.cuh", "s2_common.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libs2attn.so")


def source_hash() -> str:
    h = hashlib.sha256()
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "s2attn.h")]
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    h.update(" ".join(ARCH).encode())
    h.update(__file__.encode())
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libs2attn.so unless an up-to-date build exists.  Returns its path."""
    digest = source_hash()
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as fh:
            if fh.read().strip() == digest:
                return LIB
    nvcc = nvcc_path()
    objs = []
    tmpdir = os.path.join(PKG, "_build")
    os.makedirs(tmpdir, exist_ok=True)
    common = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                     "-I" + INCLUDE, "-I" + CSRC, "--expt-relaxed-constexpr"]
    if verbose:
        common += ["-Xptxas", "-v"]
    for src in SOURCES:
        obj = os.path.join(tmpdir, src.replace(".cu", ".o"))
        cmd = [nvcc] + common + ["-c", os.path.join(CSRC, src), "-o", obj]
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp_lib = LIB + ".tmp"
    cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp_lib] + objs
    subprocess.run(cmd, check=True)
    os.replace(tmp_lib, LIB)
    with open(STAMP, "w") as fh:
        fh.write(digest)
    return LIB


if __name__ == "__main__":
    path = build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(path)
