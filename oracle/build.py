"""Builds the CPU oracle shared library with gcc (test infrastructure)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lstm_oracle.c")
LIB_PATH = os.path.join(HERE, "liblstm_oracle.so")
LIB_PATH_SINGLE = os.path.join(HERE, "liblstm_oracle_f32.so")


def _build(path: str, defines, force: bool) -> str:
    if (not force and os.path.exists(path)
            and os.path.getmtime(path) >= os.path.getmtime(SRC)):
        return path
    tmp = path + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           *defines, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


def build(force: bool = False) -> str:
    """The oracle in IEEE double (what the tests compare the library with)."""
    return _build(LIB_PATH, [], force)


def build_single(force: bool = False) -> str:
    """The same source with every value in float (precision comparison only)."""
    return _build(LIB_PATH_SINGLE, ["-DORACLE_SINGLE"], force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
