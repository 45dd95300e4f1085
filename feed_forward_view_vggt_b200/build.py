"""Builds libvggt_attn.so in-tree with nvcc for sm_100a.

    python -m feed_forward_view_vggt_b200.build [--verbose] [--debug]

--debug builds libvggt_attn_debug.so with -DVGGT_DEBUG (device index checks).

The CUDA runtime is linked statically and the driver's tensor-map encoder
is fetched at run time, so the library loads (for symbol checks) on a
machine without a GPU driver.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libvggt_attn.so")
# -DVGGT_DEBUG: device index checks reporting through the error word
DEBUG_LIB = os.path.join(HERE, "libvggt_attn_debug.so")
SOURCES = [os.path.join(CSRC, "vggt_attn.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + \
    [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Builds the release library, or with debug=True the library with
    device index checks (-DVGGT_DEBUG); returns its path."""
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DVGGT_DEBUG"] if debug else []), "-I", INCLUDE, "-I", CSRC, "-o", tmp,
           *SOURCES]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build libvggt_attn_debug.so (-DVGGT_DEBUG)")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose, verbose=a.verbose, debug=a.debug))
