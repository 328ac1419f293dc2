"""Compile the FP64 oracle (test infrastructure) into oracle/libgdn_oracle.so.

Only the tests, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` use the oracle.  Building it is part of `__graft_entry__.build()`
so that the checker exists on every machine the tests run on.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gdn_oracle.c")
LIB = os.path.join(HERE, "libgdn_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    # -O2 without -ffast-math: the oracle keeps IEEE double semantics.
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
           "-Wall", "-Wextra", SRC, "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
