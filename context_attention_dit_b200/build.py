"""Build libcpattn.so in-tree with nvcc for sm_100a.

Usage: ``python -m context_attention_dit_b200.build`` (also called by the
repository's ``__graft_entry__.build()``).  The library is one translation unit
(``csrc/cpattn.cu``) that includes every kernel, linked against the static CUDA
runtime so that it only needs the driver at run time.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libcpattn.so")
# Debug build: every global index a kernel computes is checked against its buffer
# (-DCP_DEBUG); a violation is reported as CP_ERR_BOUNDS instead of touching memory.
LIB_DEBUG = os.path.join(PKG, "libcpattn_debug.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libcpattn.so")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    hdr = os.path.join(os.path.dirname(PKG), "include", "cpattn.h")
    return all(os.path.getmtime(s) <= t for s in sources() + [hdr, __file__])


def build(force: bool = False, verbose: bool = False, extra=(), out: str | None = None) -> str:
    """Compile csrc/cpattn.cu into ``out`` (default: the in-tree libcpattn.so)."""
    out = out or LIB
    if out == LIB and not force and up_to_date():
        return LIB
    cmd = [
        nvcc_path(), "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-cudart", "static",
        "-Xptxas", "-v" if verbose else "-O3",
        *extra,
        "-o", out + ".tmp", os.path.join(CSRC, "cpattn.cu"),
    ]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed building libcpattn.so:\n" + r.stderr[-4000:])
    os.replace(out + ".tmp", out)
    return out


def build_debug(force: bool = False) -> str:
    """Compile the bounds-checking debug library (libcpattn_debug.so)."""
    if not force and os.path.exists(LIB_DEBUG) and all(
            os.path.getmtime(s) <= os.path.getmtime(LIB_DEBUG) for s in sources() + [__file__]):
        return LIB_DEBUG
    return build(extra=("-DCP_DEBUG",), out=LIB_DEBUG)


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
    if "--debug" in sys.argv:
        print(build_debug(force=True))
