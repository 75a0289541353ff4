"""Build the trace_fp4 CUDA library in-tree (sm_100a).

    python -m fp4_block_scaled_quantizer_b200.build [--force] [--verbose] [--debug-bounds]

Produces fp4_block_scaled_quantizer_b200/libtrace_fp4.so from csrc/ with
nvcc -gencode arch=compute_100a,code=sm_100a (no fast-math: IEEE division,
reciprocal and denormals as written), static CUDA runtime.  --debug-bounds
builds libtrace_fp4_debug.so instead: the same sources with TF4_DEBUG_BOUNDS,
whose kernels check every work unit against its range and the buffers'
extent and count (rather than perform) any access outside them.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libtrace_fp4.so")
DEBUG_LIB = os.path.join(HERE, "libtrace_fp4_debug.so")
SOURCES = [os.path.join(HERE, "csrc", "trace_fp4.cu")]
DEPS = SOURCES + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + [os.path.join(ROOT, "include", "trace_fp4.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    lib = DEBUG_LIB if debug_bounds else LIB
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in DEPS):
        return lib
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC,-O2", "-shared", "-o", lib + ".tmp", *SOURCES]
    if debug_bounds:
        cmd.insert(1, "-DTF4_DEBUG_BOUNDS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                debug_bounds="--debug-bounds" in sys.argv))
