"""Builds the plain C++ CPU oracles (libsla_oracle.so: the attention operator,
the W8A8 linear layer and the gradient of the fine-tune path) with g++.

Test infrastructure: the library this builds is loaded only by the tests, the
package's smoke check and the benchmark's CPU-baseline leg (through
oracle/cpp_oracle.py).  -ffp-contract=off keeps every float32 and float64
operation a separately rounded IEEE operation, as the oracle's readings state
(and, without -ffast-math, the compiler keeps the order of every sum).

Usage: python -m oracle.build   (or build() from Python).
"""

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRCS = [os.path.join(HERE, f) for f in ("sla_oracle.cpp", "w8a8_oracle.cpp", "sla_backward_oracle.cpp")]
LIB = os.path.join(HERE, "libsla_oracle.so")


def build(force: bool = False) -> str:
    newest = max([os.path.getmtime(s) for s in SRCS] + [os.path.getmtime(__file__)])
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    cxx = os.environ.get("CXX") or shutil.which("g++") or "g++"
    tmp = LIB + ".tmp"
    subprocess.run([cxx, "-O3", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                    "-fno-fast-math", "-o", tmp] + SRCS, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
