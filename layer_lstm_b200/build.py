"""Builds liblstm_b200.so (sm_100a) in-tree with nvcc."""
from __future__ import annotations

import fcntl
import os
import subprocess
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "liblstm_b200.so")
BUILD_DIR = os.path.join(ROOT, "_build")

SOURCES = ["lstm_abi.cu", "lstm_simt.cu", "lstm_rec.cu", "lstm_tc_gemm.cu", "lstm_tc_rec.cu", "lstm_tc_rec32.cu",
           "lstm_tc_bwd.cu", "lstm_tc_bwd32.cu", "lstm_noalloc.cu"]
HEADERS = ["lstm_device.cuh", "lstm_internal.h", "lstm_tc.cuh", "lstm_tc_cluster.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "lstm.h"))
    return files


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(f) > t for f in _inputs() if os.path.exists(f))


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds the library when its sources are newer (or `force`).

    Processes that call this at the same time (the ranks of a multi-GPU
    launch, parallel test workers) build one at a time under a file lock; a
    process that got the lock after another one built finds the library
    fresh and returns."""
    if not force and not _stale():
        return LIB_PATH
    requested = time.time()
    os.makedirs(BUILD_DIR, exist_ok=True)
    with open(os.path.join(BUILD_DIR, ".lock"), "a") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        try:
            # built by another process while this one waited for the lock
            if not _stale() and (not force or os.path.getmtime(LIB_PATH) >= requested):
                return LIB_PATH
            return _compile(verbose)
        finally:
            fcntl.flock(lock, fcntl.LOCK_UN)


def _compile(verbose: bool) -> str:
    objs = []
    flags = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
             "-I", os.path.join(ROOT, "include")] + ARCH
    if verbose:
        flags += ["-Xptxas", "-v"]
    for s in SOURCES:
        obj = os.path.join(BUILD_DIR, s.replace(".cu", ".o"))
        cmd = [NVCC] + flags + ["-c", os.path.join(CSRC, s), "-o", obj]
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run([NVCC] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart"], check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
