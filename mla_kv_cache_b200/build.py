"""Build step of the kvattn shared library (libkvattn.so, sm_100a).

    python -m mla_kv_cache_b200.build            # build if sources are newer
    python -m mla_kv_cache_b200.build --force    # rebuild
    python -m mla_kv_cache_b200.build --ptxas-v  # also print registers / spills per kernel

nvcc cross-compiles for sm_100a without a GPU.  The CUDA runtime is linked statically
so the library loads on any host with the NVIDIA driver.
"""
import argparse
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkvattn.so")
HEADER = os.path.join(ROOT, "include", "kvattn.h")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--cudart=static",
    "-Xptxas=-warn-spills",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")))


def needs_build():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources() + [HEADER, __file__])


def build(force=False, ptxas_verbose=False, quiet=False):
    """Compile libkvattn.so in-tree; returns its path."""
    if not force and not ptxas_verbose and not needs_build():
        return LIB
    cmd = [NVCC] + NVCC_FLAGS + (["-Xptxas=-v"] if ptxas_verbose else []) + [
        os.path.join(CSRC, "kvattn_api.cu"), "-o", LIB + ".tmp", "-ldl"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libkvattn.so")
    os.replace(LIB + ".tmp", LIB)
    if ptxas_verbose or not quiet:
        out = (r.stdout + r.stderr).strip()
        if out:
            print(out)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_v))


if __name__ == "__main__":
    main()
