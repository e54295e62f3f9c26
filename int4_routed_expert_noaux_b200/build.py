"""Build libmoe.so (the C-ABI library of include/moe.h) in-tree for sm_100a."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
SO = os.path.join(HERE, "libmoe.so")
# the same sources with the timeline probes compiled in (-DMOE_TRACE): for
# bench.py --mode timeline only, never loaded by the library's users
SO_TRACE = os.path.join(HERE, "libmoe_trace.so")

FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
         "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) +
                  glob.glob(os.path.join(HERE, "csrc", "*.cpp")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) +
                              glob.glob(os.path.join(HERE, "csrc", "*.h")) +
                              glob.glob(os.path.join(ROOT, "include", "*.h")))


def build(force=False, verbose=False, trace=False):
    out = SO_TRACE if trace else SO
    if not force and os.path.exists(out):
        t = os.path.getmtime(out)
        if all(os.path.getmtime(d) <= t for d in deps()):
            return out
    cmd = [NVCC] + FLAGS + (["-DMOE_TRACE"] if trace else []) + [
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"), "-o", out] + sources()
    if verbose:
        cmd += ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    import sys
    build(force=True, verbose="-v" in sys.argv, trace="--trace" in sys.argv)
