"""Build libgdr.so in-tree with nvcc for sm_100a.

``python -m gated_delta_rule_recurrent_b200.build`` compiles
``csrc/gdr_api.cu`` (which includes the kernel header) into
``gated_delta_rule_recurrent_b200/libgdr.so``. A sidecar file records a hash
of every source and of the command, so ``ensure_built()`` rebuilds exactly
when something changed (file times are not trusted across copies).
"""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
REPO_DIR = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(REPO_DIR, "include")
LIB_PATH = os.path.join(PKG_DIR, "libgdr.so")
HASH_PATH = LIB_PATH + ".srchash"

SOURCES = [os.path.join(CSRC, "gdr_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, name) for name in (
    "gdr_decode.cuh", "gdr_ptx.cuh", "gdr_decode_tma.cuh", "gdr_decode_chunk.cuh", "gdr_decode_chunk_tc.cuh",
    "gdr_umma.cuh", "gdr_gate.cuh")] + [
    os.path.join(INCLUDE, "gdr.h")]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [
    "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; it is needed to build libgdr.so")


def command(extra=()) -> list:
    return [nvcc_path(), *ARCH_FLAGS, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC,
            "-o", LIB_PATH, *SOURCES]


def source_hash() -> str:
    h = hashlib.sha256()
    for path in DEPS:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode())
            h.update(f.read())
    h.update(" ".join(ARCH_FLAGS + NVCC_FLAGS).encode())
    return h.hexdigest()


def build(verbose: bool = False, extra=()) -> str:
    cmd = command(extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, flush=True)
    with open(HASH_PATH, "w") as f:
        f.write(source_hash() + "\n")
    return LIB_PATH


def is_current() -> bool:
    if not (os.path.exists(LIB_PATH) and os.path.exists(HASH_PATH)):
        return False
    with open(HASH_PATH) as f:
        return f.read().strip() == source_hash()


def ensure_built(verbose: bool = False) -> str:
    if not is_current():
        build(verbose=verbose)
    return LIB_PATH


if __name__ == "__main__":
    ptxas_info = "--ptxas-info" in sys.argv
    build(verbose=True, extra=("-Xptxas", "-v") if ptxas_info else ())
    print(LIB_PATH)
