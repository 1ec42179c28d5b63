"""Build libssd.so (the sm_100a CUDA library behind include/ssd.h) in-tree.

``python -m mamba_ssd_scan_03_b200.build`` or ``build()``.  One nvcc invocation on the single
translation unit ``csrc/ssd_lib.cu``; the .so lands next to this file so it travels with the
repository snapshot and the binding loads it from here.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libssd.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    out = [os.path.join(ROOT, "include", "ssd.h")]
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            out.append(os.path.join(CSRC, name))
    return out


def up_to_date(path, deps):
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force=False, verbose=False, ptxas_info=False):
    deps = sources()
    if not force and up_to_date(LIB, deps):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-I", os.path.join(ROOT, "include"), os.path.join(CSRC, "ssd_lib.cu"), "-o", tmp]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="-v" in sys.argv))
