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


def build(force: bool = False, verbose: bool = False, defines=(), out: str = LIB) -> str:
    """Build `out` (default: the package's librtp.so) unless it is newer than
    every source.  `defines`: extra preprocessor names, e.g. RTP_ATTN_FMA for
    the variant whose attention tiles run on the FMA pipe (a comparison build:
    give it its own `out` and load it with RTP_LIBRARY=<path>)."""
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(f) for f in _inputs())
        if os.path.getmtime(out) >= newest:
            return out
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out + f".{os.getpid()}.tmp"
    cmd = [nvcc, *NVCC_FLAGS, *[f"-D{d}" for d in defines], *[os.path.join(SRC_DIR, s) for s in SOURCES], "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    # python -m sparse_attention_decode_rtpurbo_b200.build [--force] [-v] [--define NAME ...] [--out PATH]
    argv = sys.argv[1:]
    defs = [argv[i + 1] for i, a in enumerate(argv) if a == "--define"]
    out = argv[argv.index("--out") + 1] if "--out" in argv else LIB
    print(build(force="--force" in argv, verbose="-v" in argv, defines=defs, out=os.path.abspath(out)))
