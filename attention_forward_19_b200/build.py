"""Builds libfa_fwd.so (the CUDA kernels and the C ABI) in-tree with nvcc for sm_100a.

    python -m attention_forward_19_b200.build [--force] [--ptxas-verbose] [--test-variants]

`--test-variants` also builds the test-only variants of the same source
(`TEST_VARIANTS`): the library with its lazy-rescale threshold and bf16
headroom set to zero, which is the pages' recurrence taken literally (the
reference max moves at every new maximum), and the library with branch
counters in the softmax.  Tests load them next to the product library.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "fa_fwd.cu")
DEPS = [os.path.join(PKG, "csrc", n) for n in ("fa_bwd_impl.cuh", "fa_merge_impl.cuh", "fa_proj_impl.cuh")]   # included by fa_fwd.cu
HDR = os.path.join(ROOT, "include", "fa_fwd.h")
LIB = os.path.join(PKG, "libfa_fwd.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

# name -> preprocessor definitions of a test-only build of fa_fwd.cu
TEST_VARIANTS = {
    "tau0": ("FA_RESCALE_LOG2=0", "FA_HEADROOM_LOG2=0.0f"),
    "count": ("FA_COUNT_BRANCHES=1",),
}


def variant_path(name):
    return os.path.join(PKG, f"libfa_fwd_{name}.so")


def _stale(out, sources):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force=False, verbose=False, out=LIB, defines=()):
    """Compiles fa_fwd.cu when the library is missing or older than its sources; returns its path."""
    if not force and not _stale(out, [SRC, HDR] + DEPS):
        return out
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", out, SRC]
    cmd[1:1] = [f"-D{d}" for d in defines]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    tmp = out + ".tmp"
    cmd[cmd.index(out)] = tmp
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build_variant(name, force=False):
    """Builds one of TEST_VARIANTS (test infrastructure, not the product library); returns its path."""
    return build(force=force, out=variant_path(name), defines=TEST_VARIANTS[name])


if __name__ == "__main__":
    force = "--force" in sys.argv
    print(build(force=force, verbose="--ptxas-verbose" in sys.argv))
    if "--test-variants" in sys.argv:
        for n in TEST_VARIANTS:
            print(build_variant(n, force=force))
