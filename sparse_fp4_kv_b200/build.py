"""Build libcsa2.so in-tree with nvcc for sm_100a.

    python -m sparse_fp4_kv_b200.build [--force]

One translation unit (csrc/csa2.cu includes every kernel). The CUDA runtime
is linked statically and the driver entry point for tensor-map encoding is
fetched at run time, so the library loads on a machine without a GPU.
No fast-math: the quantiser's divisions and comparisons must be IEEE.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "csa2.cu")
LIB = os.path.join(HERE, "libcsa2.so")
# the tensor-core rate probe used by the measurement (bench.py), not the path
PEAK_SRC = os.path.join(HERE, "csrc", "peak.cu")
PEAK_LIB = os.path.join(HERE, "libcsa2_peak.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "-cudart", "static"]


def _inputs():
    return glob.glob(os.path.join(HERE, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def _compile(src, lib, force, verbose):
    if (not force and os.path.exists(lib)
            and all(os.path.getmtime(lib) >= os.path.getmtime(f) for f in _inputs())):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-o", lib + ".tmp", src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    _compile(PEAK_SRC, PEAK_LIB, force, verbose)
    return _compile(SRC, LIB, force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
