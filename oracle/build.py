"""Compile the CPU oracle (test infrastructure) into oracle/liboracle.so.

Plain g++, no CUDA.  -ffp-contract=off keeps every fp32 operation rounded on
its own, as the oracle's definitions state.
"""
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")


def _digest() -> str:
    with open(SRC, "rb") as f:
        return hashlib.sha256(f.read() + open(__file__, "rb").read()).hexdigest()


def build(force: bool = False) -> str:
    stamp = LIB + ".stamp"
    if not force and os.path.exists(LIB) and os.path.exists(stamp) and open(stamp).read().strip() == _digest():
        return LIB
    cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    with open(stamp, "w") as f:
        f.write(_digest())
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
