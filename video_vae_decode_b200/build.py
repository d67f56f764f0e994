"""Build libqvae.so (the CUDA path) in-tree for sm_100a.

    python -m video_vae_decode_b200.build            # libqvae.so
    python -m video_vae_decode_b200.build --debug    # libqvae_debug.so: bounds-checked loads and stores

The debug library compiles the kernels' bounds checks in (-DQVAE_DEBUG_CHECKS):
every TMA load's and store's coordinates and shared-memory range, every
direct store's index and every MMA's accumulator columns are checked before
the access; a failed check is recorded (qvae_get_error() returns
QVAE_ERR_BOUNDS) and the access skipped.  It exports the same C ABI.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqvae.so")
LIB_DEBUG = os.path.join(HERE, "libqvae_debug.so")
ROOT = os.path.dirname(HERE)
SOURCES = ["qvae.cu"]
DEPS = ["qvae.cu", "conv.cuh", "quant.cuh", "ptx.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def command(out: str, extra=()):
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
            "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", os.path.join(ROOT, "include"), *extra,
            *[os.path.join(CSRC, s) for s in SOURCES], "-o", out]


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    newest = max(os.path.getmtime(os.path.join(CSRC, d)) for d in DEPS)
    newest = max(newest, os.path.getmtime(os.path.join(ROOT, "include", "qvae.h")))
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest:
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    extra = (["-Xptxas", "-v"] if verbose else []) + (["-DQVAE_DEBUG_CHECKS"] if debug else [])
    subprocess.run(command(tmp, extra), check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
