"""Builds libpagedkv.so in-tree with nvcc for sm_100a.

One shared library: the CUDA translation unit (all kernels + device C-ABI
entry points) and the host C++ block manager / scheduler. CUDA runtime is
linked statically; only the pa_* symbols are exported. A digest of the sources
and flags is stored beside the library; build() rebuilds only when it changes.
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
LIB = os.path.join(PKG, "libpagedkv.so")
STAMP = LIB + ".digest"

SOURCES = [
    os.path.join(CSRC, "device", "pagedkv_device.cu"),
    os.path.join(CSRC, "host", "block_manager.cpp"),
    os.path.join(CSRC, "host", "scheduler.cpp"),
]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpagedkv.so")


def _digest(extra) -> str:
    h = hashlib.sha256()
    files = [os.path.join(INCLUDE, "pagedkv.h")]
    for d, _, names in os.walk(CSRC):
        files += [os.path.join(d, n) for n in names]
    for f in sorted(files):
        h.update(os.path.relpath(f, ROOT).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(ARCH + FLAGS + list(extra)).encode())
    return h.hexdigest()


def command(extra=()) -> list:
    return ([nvcc_path()] + ARCH + FLAGS + list(extra) + ["-I", INCLUDE,
            "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
            "-o", LIB] + SOURCES)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    digest = _digest(extra)
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() == digest:
                return LIB
    cmd = command(extra)
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    tmp = LIB + ".tmp"
    cmd[cmd.index("-o") + 1] = tmp
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed building libpagedkv.so:\n" + r.stdout + r.stderr)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(digest + "\n")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
