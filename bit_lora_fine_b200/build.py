"""Builds libfourtune.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m bit_lora_fine_b200.build [--verbose]

Every kernel is compiled for sm_100a only (tcgen05 / TMA instructions); the
library links the CUDA runtime statically and reaches the driver's tensor-map
encoder through cudaGetDriverEntryPoint, so it needs no libcuda at link time.
"""
import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libfourtune.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.h")) + glob.glob(os.path.join(PKG, "csrc", "*.cuh")) +
                  glob.glob(os.path.join(ROOT, "include", "fourtune", "*.h")))


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in sources() + headers() + [__file__])


def build(verbose=False, force=False):
    if not force and up_to_date():
        return LIB
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           "-Xcompiler", "-Wall", "-o", LIB + ".tmp"] + sources()
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(verbose=a.verbose, force=a.force or a.verbose))
    sys.exit(0)
