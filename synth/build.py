"""Build the seeded input generator: libsynth.so (host, gcc) and
libsynth_dev.so (device, nvcc for sm_100a)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force=False, device=True):
    host_src = [os.path.join(HERE, "synth.c"), os.path.join(HERE, "synth_core.h"),
                os.path.join(HERE, "synth.h")]
    host_so = os.path.join(HERE, "libsynth.so")
    if force or _stale(host_so, host_src):
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
             "-std=c11", "-Wall", "-o", host_so, host_src[0], "-lm"])
    if device:
        dev_src = [os.path.join(HERE, "synth_dev.cu"), os.path.join(HERE, "synth_core.h")]
        dev_so = os.path.join(HERE, "libsynth_dev.so")
        if force or _stale(dev_so, dev_src):
            subprocess.check_call(
                [NVCC, "-O3", "-shared", "-Xcompiler", "-fPIC",
                 "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                 "-fmad=false", "-o", dev_so, dev_src[0]])


if __name__ == "__main__":
    build(force=True)
