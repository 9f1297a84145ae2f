"""Build libuf.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

Usage: python block_sparse_causal_b200/build.py [--force] [--ptxas-v]

Run by path (or loaded with ``load_builder``): importing the package itself
loads libuf.so, which must exist first.

Build identity: the SHA-256 of the library's sources (csrc/ and include/) is
compiled into the library (``uf_source_hash()``) and written beside it
(``libuf.so.srchash``).  A build is reused only while that hash matches the
tree; the binding refuses a library built from other sources.

Register check: the attention kernel splits its launch registers between
warpgroups, a split that only holds for the count it was written for, so the
build reads ptxas' resource report and fails when any attention kernel was
compiled to another count.
"""
from __future__ import annotations

import hashlib
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libuf.so")
HASH_FILE = LIB + ".srchash"

# registers per thread the attention kernel's warpgroup split is written for
# (ATTN_LAUNCH_REGS in csrc/attention.cuh)
ATTN_LAUNCH_REGS = 168

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-v",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libuf.so")


def _sources():
    files = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh", ".h"))]
    files.append(os.path.join(INCLUDE, "uf.h"))
    return files


def source_hash() -> str:
    """First 16 hex digits of the SHA-256 over the sources' names and bytes."""
    h = hashlib.sha256()
    for f in _sources():
        h.update(os.path.relpath(f, ROOT).encode())
        h.update(b"\0")
        with open(f, "rb") as fh:
            h.update(fh.read())
        h.update(b"\0")
    return h.hexdigest()[:16]


def built_hash() -> str | None:
    """Source hash recorded by the last build, or None."""
    if not os.path.exists(LIB) or not os.path.exists(HASH_FILE):
        return None
    with open(HASH_FILE) as f:
        return f.read().strip() or None


def up_to_date() -> bool:
    return built_hash() == source_hash()


def check_attention_registers(ptxas_report: str) -> None:
    """Fail when an attention kernel was compiled to a register count other
    than the one its warpgroup split adds up to."""
    found = 0
    for m in re.finditer(r"Compiling entry function '(\w*attn_kernel\w*)'.*?Used (\d+) registers", ptxas_report,
                         flags=re.S):
        found += 1
        if int(m.group(2)) != ATTN_LAUNCH_REGS:
            raise RuntimeError(f"{m.group(1)} compiled to {m.group(2)} registers per thread; its warpgroup "
                               f"register split needs exactly {ATTN_LAUNCH_REGS}")
    if found == 0:
        raise RuntimeError("no attention kernel in ptxas' resource report")


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    """Compile csrc/uf.cu into block_sparse_causal_b200/libuf.so, unless the
    library on disk was built from the same sources."""
    want = source_hash()
    if not force and built_hash() == want:
        if verbose:
            print(f"libuf.so up to date (source hash {want}): reused", flush=True)
        return LIB
    tmp = LIB + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, *extra_flags, f"-DUF_SOURCE_HASH=\"{want}\"", "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, os.path.join(CSRC, "uf.cu")]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    report = res.stdout + res.stderr
    check_attention_registers(report)
    if verbose and "--ptxas-v" in sys.argv:
        print(report, flush=True)
    os.replace(tmp, LIB)
    with open(HASH_FILE, "w") as f:
        f.write(want + "\n")
    if verbose:
        print(f"libuf.so compiled (source hash {want})", flush=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
