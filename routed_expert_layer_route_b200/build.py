"""Build libmoe.so (the C-ABI library) for B200, sm_100a, in-tree, and its
checked twin libmoe_checks.so (compiled with MOE_CHECKS=1: kernels also
verify the index tables they otherwise trust and record MOE_ERR_DEVICE_CHECK).

    python -m routed_expert_layer_route_b200.build [--force] [--checks]

The library is one translation unit (csrc/moe_api.cu includes the kernel
headers).  Routing arithmetic is written with explicit round-to-nearest
intrinsics, so no global floating-point flags are needed for bit-exactness;
fast-math is never used.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libmoe.so")
LIB_CHECKS = os.path.join(HERE, "libmoe_checks.so")
MAIN = os.path.join(CSRC, "moe_api.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3",
    "-lineinfo",
    "-std=c++17",
    "-Xcompiler", "-fPIC",
    "-shared",
]


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date(lib=LIB):
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force=False, verbose=False, checks=False):
    """Compile libmoe.so (checks: libmoe_checks.so) if any source is newer;
    return its path."""
    lib = LIB_CHECKS if checks else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [nvcc()] + NVCC_FLAGS + (["-DMOE_CHECKS=1"] if checks else []) + ["-o", tmp, MAIN]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                checks="--checks" in sys.argv))
