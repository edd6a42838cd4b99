"""Build the sm_100a shared library ``libgdn.so`` in this package directory.

    python -m frame_wise_gated_deltanet_b200.build [--verbose-ptxas] [--debug]

nvcc cross-compiles for sm_100a without a GPU. The CUDA runtime is linked statically and the
driver's tensor-map encoder is looked up at run time, so the library loads on a machine with
no GPU driver (every call then returns GDN_ERR_CUDA).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libgdn.so")
DEBUG_LIB = os.path.join(HERE, "libgdn_debug.so")  # -DGDN_DEBUG: device-side copy checks
SOURCES = [os.path.join(HERE, "csrc", "gdn_api.cu")]
DEPENDS = SOURCES + [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libgdn.so")


def command(verbose_ptxas: bool = False, debug: bool = False) -> list:
    cmd = [
        nvcc_path(), "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
        "-I", os.path.join(os.path.dirname(HERE), "include"),
        "-o", DEBUG_LIB if debug else LIB,
    ] + (["-DGDN_DEBUG"] if debug else []) + SOURCES
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in DEPENDS if os.path.exists(f))


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    """Build libgdn.so, or with debug=True libgdn_debug.so (the device-side checks)."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not verbose_ptxas and up_to_date(lib):
        return lib
    cmd = command(verbose_ptxas, debug)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose_ptxas:
        sys.stderr.write(r.stdout + r.stderr)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true",
                    help="build libgdn_debug.so (device-side copy and address checks)")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, debug=a.debug))
