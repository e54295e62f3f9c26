"""Build the fp64 CPU oracle (liboracle.so).  Test infrastructure only."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build(force=False):
    src = [os.path.join(HERE, "oracle.c"), os.path.join(HERE, "oracle.h")]
    so = os.path.join(HERE, "liboracle.so")
    if force or not os.path.exists(so) or any(
            os.path.getmtime(s) > os.path.getmtime(so) for s in src):
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
             "-std=c11", "-Wall", "-o", so, src[0], "-lm"])
    return so


if __name__ == "__main__":
    build(force=True)
