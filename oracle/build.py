"""Build the CPU oracle shared library (test infrastructure only).

g++ -O2 -ffp-contract=off, no fast-math: every float operation in the oracle
rounds exactly as written.  The result, ``oracle/libstq_oracle.so``, is loaded
only by tests, ``__graft_entry__.smoke()`` and bench.py's CPU legs.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = [os.path.join(HERE, "stq_oracle.cpp")]
HEADERS = [os.path.join(HERE, "stq_oracle.h")]
LIB = os.path.join(HERE, "libstq_oracle.so")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS + [__file__])


def build(force: bool = False) -> str:
    if force or _stale():
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp] + SOURCES
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
