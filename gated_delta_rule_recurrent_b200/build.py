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
# A second build with -DGDR_TEST_HOOKS, for the failure-path tests only: the
# same kernels with a shortened budget for abandonable waits and a switch that
# holds one tile back. The shipped libgdr.so never contains the hooks.
TEST_HOOKS_LIB_PATH = os.path.join(PKG_DIR, "libgdr_testhooks.so")
TEST_HOOKS_FLAGS = ["-DGDR_TEST_HOOKS"]

SOURCES = [os.path.join(CSRC, "gdr_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, name) for name in (
    "gdr_decode.cuh", "gdr_ptx.cuh", "gdr_decode_tma.cuh", "gdr_decode_chunk.cuh", "gdr_decode_chunk_tc.cuh",
    "gdr_decode_rows.cuh",
    "gdr_umma.cuh", "gdr_gate.cuh", "gdr_prefill_tc.cuh")] + [
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


def command(extra=(), out=LIB_PATH) -> list:
    return [nvcc_path(), *ARCH_FLAGS, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC,
            "-o", out, *SOURCES]


def source_hash(flags=()) -> str:
    h = hashlib.sha256()
    for path in DEPS:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode())
            h.update(f.read())
    h.update(" ".join(ARCH_FLAGS + NVCC_FLAGS + list(flags)).encode())
    return h.hexdigest()


def build(verbose: bool = False, extra=(), test_hooks: bool = False) -> str:
    out = TEST_HOOKS_LIB_PATH if test_hooks else LIB_PATH
    flags = TEST_HOOKS_FLAGS if test_hooks else []
    cmd = command([*flags, *extra], out)
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, flush=True)
    with open(out + ".srchash", "w") as f:
        f.write(source_hash(flags) + "\n")
    return out


def is_current(test_hooks: bool = False) -> bool:
    out = TEST_HOOKS_LIB_PATH if test_hooks else LIB_PATH
    if not (os.path.exists(out) and os.path.exists(out + ".srchash")):
        return False
    with open(out + ".srchash") as f:
        return f.read().strip() == source_hash(TEST_HOOKS_FLAGS if test_hooks else [])


def ensure_built(verbose: bool = False, test_hooks: bool = False) -> str:
    if not is_current(test_hooks):
        build(verbose=verbose, test_hooks=test_hooks)
    return TEST_HOOKS_LIB_PATH if test_hooks else LIB_PATH


if __name__ == "__main__":
    ptxas_info = "--ptxas-info" in sys.argv
    hooks = "--test-hooks" in sys.argv
    print(build(verbose=True, extra=("-Xptxas", "-v") if ptxas_info else (), test_hooks=hooks))
