"""Builds the C++ oracle (oracle/dsa_oracle.cpp) into oracle/libdsa_oracle_cpp.so with g++.

    python -m oracle.build_cpp

Test infrastructure only: the library is loaded by oracle/cpp_oracle.py for the tests, the
smoke check and the benchmark's CPU baseline. -ffp-contract=off keeps every multiply and add
a separate IEEE double operation, in the order the source states.
"""

from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dsa_oracle.cpp")
LIB = os.path.join(HERE, "libdsa_oracle_cpp.so")
FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["g++"] + FLAGS + [SRC, "-o", LIB]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"g++ failed for the C++ oracle:\n{res.stdout}\n{res.stderr}")
    return LIB


if __name__ == "__main__":
    print(build(force=True))
