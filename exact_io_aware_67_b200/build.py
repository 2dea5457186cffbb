"""Build step: compile libfa.so (all CUDA kernels + the C ABI) for sm_100a.

    python -m exact_io_aware_67_b200.build [--force] [--verbose]

Runs nvcc once over ``csrc/fa_api.cu`` (the kernels are header templates
included there) and writes ``libfa.so`` next to this file, where the Python
binding loads it.  ``--verbose`` adds ``-Xptxas -v`` (registers, spills,
shared memory per kernel).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfa.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _sources():
    out = [os.path.join(INCLUDE, "fa.h")]
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(CSRC, f))
    return out


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def nvcc_command(out, verbose=False):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, "-o", out, os.path.join(CSRC, "fa_api.cu")]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    return cmd


def build(force=False, verbose=False):
    if not force and not _stale():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.run(nvcc_command(tmp, verbose), check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
