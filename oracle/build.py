"""Compile the CPU oracle (plain C) into ``oracle/liboracle.so``.

Test infrastructure: the oracle is built beside the CUDA library so that the
test suite, the smoke check and the benchmark's CPU baseline can load it.
Strict IEEE flags: no fast-math, no contraction into fused multiply-adds.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(OUT)
            and os.path.getmtime(OUT) >= max(os.path.getmtime(SRC),
                                             os.path.getmtime(os.path.join(HERE, "oracle.h")))):
        return OUT
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
           "-o", OUT + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
