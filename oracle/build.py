"""Compile the CPU oracle into ``liboracle.so`` (plain C, OpenMP, no FMA contraction).

Part of the test infrastructure; run by ``__graft_entry__.build()`` and on first use.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))


def build(verbose: bool = False) -> str:
    src = os.path.join(HERE, "qnt_oracle.c")
    out = os.path.join(HERE, "liboracle.so")
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-o", out, src, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
