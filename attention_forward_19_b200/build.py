"""Builds libfa_fwd.so (the CUDA kernels and the C ABI) in-tree with nvcc for sm_100a.

    python -m attention_forward_19_b200.build [--force] [--ptxas-verbose]
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "fa_fwd.cu")
DEPS = [os.path.join(PKG, "csrc", n) for n in ("fa_bwd_impl.cuh", "fa_bwd_atomic_impl.cuh", "fa_merge_impl.cuh",
                                            "fa_proj_impl.cuh")]   # included by fa_fwd.cu
HDR = os.path.join(ROOT, "include", "fa_fwd.h")
LIB = os.path.join(PKG, "libfa_fwd.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale(out, sources):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force=False, verbose=False, out=LIB):
    """Compiles fa_fwd.cu when the library is missing or older than its sources; returns its path."""
    if not force and not _stale(out, [SRC, HDR] + DEPS):
        return out
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", out, SRC]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    tmp = out + ".tmp"
    cmd[cmd.index(out)] = tmp
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--ptxas-verbose" in sys.argv))
