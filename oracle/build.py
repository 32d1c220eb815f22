"""Build the oracle's shared library (test infrastructure only).

Compiles ``h3_oracle.cpp`` with the host C++ compiler into
``oracle/_lib/libh3_oracle.so``. -O3 without fast-math (no floating-point reassociation), so the float
division and round-half-even steps of the quantizer follow IEEE binary32.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "h3_oracle.cpp")
OUT_DIR = os.path.join(HERE, "_lib")
OUT = os.path.join(OUT_DIR, "libh3_oracle.so")


def build(force: bool = False) -> str:
    os.makedirs(OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(OUT)
            and os.path.getmtime(OUT) >= os.path.getmtime(SRC)):
        return OUT
    # x86-64-v3 (AVX2) keeps the library loadable on any recent x86 host.
    cmd = ["g++", "-O3", "-march=x86-64-v3", "-fno-fast-math", "-ffp-contract=off",
           "-fopenmp", "-fPIC", "-shared", "-std=c++17", SRC, "-o", OUT + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
