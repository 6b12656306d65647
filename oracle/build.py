"""Compiles the CPU oracle into ``oracle/liboracle.so``.

Test infrastructure: the oracle is built so that tests, the smoke check and
the benchmark's CPU baseline can call it; the product path never does.
Flags: no fast-math and no implicit FMA contraction, so the binary32 steps run
exactly in the order the source writes them.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["g++", "-O2", "-ffp-contract=off", "-fno-fast-math", "-frounding-math", "-fopenmp",
           "-shared", "-fPIC", "-Wall", "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
