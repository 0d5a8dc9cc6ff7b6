"""Builds libs2attn.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m sparse_attention_attn_b200.build          # build if sources changed
    python -m sparse_attention_attn_b200.build --force  # always rebuild
    python -m sparse_attention_attn_b200.build --debug  # libs2attn_debug.so: kernels with index checks

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
LIB_DEBUG = os.path.join(PKG, "libs2attn_debug.so")

SOURCES = ["s2attn.cu", "s2_fwd.cu", "s2_fwd64.cu", "s2_bwd.cu", "s2_bwd_fused.cu", "s2_rope.cu", "s2_segment.cu", "s2_nf4.cu", "s2_bwd_ds.cu", "s2_bwd_kv128.cu"]
HEADERS = ["s2_ptx.cuh", "s2_common.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libs2attn.so")


def source_hash(debug: bool = False) -> str:
    h = hashlib.sha256()
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "s2attn.h")]
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    h.update(" ".join(ARCH).encode())
    h.update(__file__.encode())
    h.update(b"debug" if debug else b"release")
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile libs2attn.so (or, with debug, libs2attn_debug.so: the same
    sources with the kernels' index checks compiled in) unless an up-to-date
    build exists.  Returns its path.  The sources compile in parallel."""
    lib = LIB_DEBUG if debug else LIB
    stamp = lib + ".srchash"
    digest = source_hash(debug)
    if not force and os.path.exists(lib) and os.path.exists(stamp):
        with open(stamp) as fh:
            if fh.read().strip() == digest:
                return lib
    nvcc = nvcc_path()
    tmpdir = os.path.join(PKG, "_build_debug" if debug else "_build")
    os.makedirs(tmpdir, exist_ok=True)
    common = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                     "-I" + INCLUDE, "-I" + CSRC, "--expt-relaxed-constexpr"]
    if debug:
        common += ["-DS2ATTN_DEBUG_CHECKS"]
    if verbose:
        common += ["-Xptxas", "-v"]
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(tmpdir, src.replace(".cu", ".o"))
        procs.append((src, subprocess.Popen([nvcc] + common + ["-c", os.path.join(CSRC, src), "-o", obj])))
        objs.append(obj)
    failed = [src for src, p in procs if p.wait() != 0]
    if failed:
        raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
    tmp_lib = lib + ".tmp"
    cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp_lib] + objs
    subprocess.run(cmd, check=True)
    os.replace(tmp_lib, lib)
    with open(stamp, "w") as fh:
        fh.write(digest)
    return lib


if __name__ == "__main__":
    path = build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv)
    print(path)
