"""Builds the fp64 CPU oracle (test infrastructure) into oracle/_build/libhils_oracle.so.

Plain gcc, -O2, no fast-math: the oracle's arithmetic must stay IEEE fp64 in program order.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
BUILD_DIR = os.path.join(HERE, "_build")
LIB_PATH = os.path.join(BUILD_DIR, "libhils_oracle.so")
SOURCES = [os.path.join(HERE, "hils_oracle.c"), os.path.join(HERE, "hils_oracle_bwd.c"),
           os.path.join(HERE, "hils_oracle_prologue.c")]
HEADERS = [os.path.join(HERE, "hils_oracle.h")]


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(s) > t for s in SOURCES + HEADERS + [__file__])


def build(force: bool = False) -> str:
    if force or _stale():
        os.makedirs(BUILD_DIR, exist_ok=True)
        tmp = LIB_PATH + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", "-Wall", "-Wextra",
               "-fno-fast-math", "-ffp-contract=off", "-o", tmp] + SOURCES + ["-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
