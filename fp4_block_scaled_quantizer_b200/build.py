"""Build the trace_fp4 CUDA library in-tree (sm_100a).

    python -m fp4_block_scaled_quantizer_b200.build [--force] [--verbose]

Produces fp4_block_scaled_quantizer_b200/libtrace_fp4.so from csrc/ with
nvcc -gencode arch=compute_100a,code=sm_100a (no fast-math: IEEE division,
reciprocal and denormals as written), static CUDA runtime.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libtrace_fp4.so")
SOURCES = [os.path.join(HERE, "csrc", "trace_fp4.cu")]
DEPS = SOURCES + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + [os.path.join(ROOT, "include", "trace_fp4.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in DEPS):
        return LIB
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC,-O2", "-shared", "-o", LIB + ".tmp", *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
