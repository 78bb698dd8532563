"""Compiles the CPU oracle (dsa_oracle.c) into liboracle.so beside it.

The oracle is test infrastructure: only the tests, the smoke check and the
benchmark's CPU-baseline leg load it."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dsa_oracle.c")
LIB_PATH = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC)):
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    # -O2 without -ffast-math: the fp64 softmax keeps IEEE semantics.
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"])
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True))
