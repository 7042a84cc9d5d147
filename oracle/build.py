"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so.

Plain g++ with OpenMP.  -ffp-contract=off keeps every multiply and add a
separately rounded IEEE operation, as the oracle's definitions require.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "m3_oracle.cpp")
SRCS = [SRC, os.path.join(HERE, "dit_oracle.cpp")]
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and \
            os.path.getmtime(OUT) >= max(os.path.getmtime(f) for f in SRCS):
        return OUT
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", *SRCS, "-o", OUT + ".tmp"]
    subprocess.check_call(cmd)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
