"""Compile the C part of the oracle (test infrastructure; see ripe_oracle.py).

Run as ``python oracle/build.py``; the package build calls ``build_oracle()``.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "libripe_oracle.so")
SRC = os.path.join(HERE, "ripe_oracle.c")


def build_oracle(force: bool = False) -> str:
    if force or not os.path.exists(SO) or os.path.getmtime(SO) < os.path.getmtime(SRC):
        tmp = SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-Wall",
                               "-o", tmp, SRC, "-lm"])
        os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build_oracle(force=True))
