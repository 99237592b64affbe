"""Compile the fp64 CPU oracle (``oracle.c``) into ``liboracle.so`` beside it.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline load the result.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, SRC, "-lm"]
    )
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
