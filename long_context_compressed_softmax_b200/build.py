"""Build liblcsa.so in place (sm_100a).

    python -m long_context_compressed_softmax_b200.build [--verbose]

Compiles csrc/lcsa.cu (the translation unit that includes every kernel) and
csrc/noalloc.cu with nvcc for sm_100a and writes liblcsa.so next to this file.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "liblcsa.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I" + os.path.join(ROOT, "include"),
    "-I" + SRC,
]


def sources():
    return sorted(os.path.join(SRC, f) for f in os.listdir(SRC) if f.endswith((".cu", ".cuh")))


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    deps = sources() + [os.path.join(ROOT, "include", "lcsa.h"), __file__]
    return all(os.path.getmtime(p) <= t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    tmp = OUT + ".tmp"
    units = [os.path.join(SRC, "lcsa.cu"), os.path.join(SRC, "noalloc.cu")]
    cmd = [nvcc, *NVCC_FLAGS, "-o", tmp, *units]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv or "--verbose" in sys.argv, verbose="--verbose" in sys.argv)
    print(OUT)
