"""Compiles ``oracle/attn_oracle.c`` and ``oracle/attn_bwd_oracle.c`` into
``oracle/liboracle.so`` with gcc.

Plain IEEE fp64 (no -ffast-math), pthreads.  Test infrastructure only.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attn_oracle.c")
SRC_BWD = os.path.join(HERE, "attn_bwd_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force=False, verbose=False):
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(SRC_BWD))):
        return LIB
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
           "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, SRC_BWD, "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
