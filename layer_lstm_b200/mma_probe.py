"""Builds and runs the tcgen05.mma issue-cost probe (csrc/mma_issue_probe.cu).

    python -m layer_lstm_b200.mma_probe            # CSV on stdout; needs a B200

A measurement tool beside the library, not part of it: it shows that a
chain of M = 128 (or 64), K = 16 bf16 MMAs costs the same per instruction for
every N from 16 to 256, which is why the tensor-core recurrence is planned by
its MMA instruction count per step.
"""
import os
import subprocess
import sys
import tempfile

from . import build as _build

SRC = os.path.join(_build.CSRC, "mma_issue_probe.cu")


def main() -> int:
    exe = os.path.join(tempfile.mkdtemp(prefix="mma_probe_"), "mma_issue_probe")
    subprocess.run([_build.NVCC, "-O2"] + _build.ARCH + ["-o", exe, SRC], check=True)
    return subprocess.run([exe]).returncode


if __name__ == "__main__":
    sys.exit(main())
