"""Builds ``scatter_gemm_b200/liblora_sgmv.so`` (sm_100a) with nvcc, in-tree.

The library links the CUDA runtime statically and resolves driver entry
points at run time, so it loads (and exports its symbols) on a machine
without a GPU driver; calls that need the device then return LORA_ERR_CUDA.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblora_sgmv.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-fvisibility=hidden,-Wall,-Wextra",
    "-shared", "-cudart", "static",
    "-Werror", "all-warnings",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return (sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
            + [os.path.join(ROOT, "include", "lora_sgmv.h"), __file__])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [NVCC] + FLAGS + ["-I", os.path.join(ROOT, "include")] + sources() + \
          ["-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
