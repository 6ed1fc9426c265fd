"""Builds the CPU oracle library ``oracle/liboracle.so`` with g++.

Strict IEEE arithmetic: no FMA contraction, no fast-math.  Test
infrastructure only (see ``oracle/__init__.py``).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")


def build_oracle(verbose=False):
    src = os.path.join(HERE, "oracle.cpp")
    tmp = LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-pthread", "-Wall", "-o", tmp, src]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build_oracle(verbose=True))
