"""Compile the CUDA sources into librtp.so (sm_100a), in the package directory."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "librtp.so")
SOURCES = ["rtp_decode.cu"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include")]


def _inputs():
    files = [os.path.join(SRC_DIR, f) for f in os.listdir(SRC_DIR)]
    files.append(os.path.join(ROOT, "include", "rtp_decode.h"))
    return files


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(f) for f in _inputs())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc, *NVCC_FLAGS, *[os.path.join(SRC_DIR, s) for s in SOURCES], "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
