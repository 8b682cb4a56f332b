"""Build libnvfp4.so in-tree with nvcc for sm_100a.

    python -m nvfp4_w4a4_quantized_05_b200.build [--force] [--verbose]

Flags: -gencode arch=compute_100a,code=sm_100a (tcgen05 / TMA need the
architecture-specific target), -lineinfo for profiling, -fmad=false so the
quantizer's multiply-then-round steps never fuse into FMAs, static cudart.
The driver API (tensor-map encoding) is reached through
cudaGetDriverEntryPoint, so libcuda is not linked.
"""
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvfp4.so")
STAMP = LIB + ".srchash"
SOURCES = ["api.cu", "quant.cu", "gemm.cu", "w4a16.cu"]
HEADERS = ["ptx.cuh", "internal.h"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _src_hash() -> str:
    h = hashlib.sha256()
    for f in SOURCES + HEADERS:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    with open(os.path.join(ROOT, "include", "nvfp4.h"), "rb") as fh:
        h.update(fh.read())
    h.update(" ".join(FLAGS).encode())
    return h.hexdigest()


def needs_build() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(STAMP):
        return True
    with open(STAMP) as f:
        return f.read().strip() != _src_hash()


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, "-shared", "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(_src_hash())
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
