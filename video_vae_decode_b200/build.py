"""Build libqvae.so (the CUDA path) in-tree for sm_100a.

    python -m video_vae_decode_b200.build
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqvae.so")
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


def build(force: bool = False, verbose: bool = False) -> str:
    newest = max(os.path.getmtime(os.path.join(CSRC, d)) for d in DEPS)
    newest = max(newest, os.path.getmtime(os.path.join(ROOT, "include", "qvae.h")))
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    extra = ["-Xptxas", "-v"] if verbose else []
    subprocess.run(command(tmp, extra), check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
