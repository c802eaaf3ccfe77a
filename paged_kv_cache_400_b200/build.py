"""Builds libpagedkv.so in-tree with nvcc for sm_100a.

One shared library: the CUDA translation unit (all kernels + device C-ABI
entry points) and the host C++ block manager / scheduler. CUDA runtime is
linked statically; only the pa_* symbols are exported. A digest of the sources
and flags is stored beside the library; build() rebuilds only when it changes.

Comparison builds (build(variant=...)) compile the same sources with one
compile-time switch into a library of their own, libpagedkv_<variant>.so; the
product library never contains their kernels:
  prefill_mma_sync   pa_prefill runs the mma.sync prefill kernel
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
VARIANTS = {
    "prefill_mma_sync": ["-DPA_PREFILL_MMA_SYNC"],
}
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


def lib_path(variant=None) -> str:
    """The product library, or a comparison build's library."""
    if variant is None:
        return LIB
    if variant not in VARIANTS:
        raise ValueError(f"unknown build variant {variant!r} (one of {sorted(VARIANTS)})")
    return os.path.join(PKG, f"libpagedkv_{variant}.so")


def command(extra=(), out=LIB) -> list:
    return ([nvcc_path()] + ARCH + FLAGS + list(extra) + ["-I", INCLUDE,
            "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
            "-o", out] + SOURCES)


def build(force: bool = False, verbose: bool = False, extra=(), variant=None) -> str:
    out = lib_path(variant)
    flags = list(extra) + (VARIANTS[variant] if variant else [])
    stamp = out + ".digest"
    digest = _digest(flags)
    if not force and os.path.exists(out) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == digest:
                return out
    cmd = command(flags, out)
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    tmp = out + ".tmp"
    cmd[cmd.index("-o") + 1] = tmp
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed building {os.path.basename(out)}:\n" + r.stdout + r.stderr)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(tmp, out)
    with open(stamp, "w") as f:
        f.write(digest + "\n")
    return out


if __name__ == "__main__":
    names = [a[len("--variant="):] for a in sys.argv[1:] if a.startswith("--variant=")]
    for v in (names or [None]):
        print(build(force="--force" in sys.argv, verbose=True, variant=v))
