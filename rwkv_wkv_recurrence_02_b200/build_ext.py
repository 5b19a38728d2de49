"""Build libwkv.so (the sm_100a CUDA library behind include/wkv.h) in-tree.

nvcc cross-compiles for sm_100a without a GPU, so this runs on any machine
with the CUDA 12.9 toolkit.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libwkv.so")
SOURCES = [os.path.join(CSRC, "wkv_api.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + \
    [os.path.join(ROOT, "include", "wkv.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA 12.9 toolkit is required to build libwkv.so")


def build_command(out: str, extra=()):
    return [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
            "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-warn-spills", *extra, "-o", out, *SOURCES]


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libwkv.so if it is missing or older than any source; return its path."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(p) <= t for p in DEPENDS):
            return LIB
    tmp = LIB + ".tmp"
    cmd = build_command(tmp, ("-Xptxas", "-v") if verbose else ())
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
