"""Concurrent builds of the library are serialised (CPU).

The ranks of a multi-GPU launch each load the library and build it if its
sources look newer; two nvcc runs writing the same object files at once
would corrupt them.  Two processes build at the same time into a temporary
directory with a stand-in compiler that logs each invocation: exactly one
full build must run, and a later call must find the library fresh.
"""
import os
import stat
import subprocess
import sys
import textwrap

from layer_lstm_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FAKE_NVCC = textwrap.dedent("""\
    #!/bin/bash
    out=""
    while [ $# -gt 0 ]; do
      if [ "$1" = "-o" ]; then out="$2"; shift; fi
      shift
    done
    echo "$out" >> "$FAKE_NVCC_LOG"
    sleep 0.2
    : > "$out"
    """)

CHILD = textwrap.dedent("""\
    import os, sys
    sys.path.insert(0, {root!r})
    from layer_lstm_b200 import build as b
    b.LIB_PATH = os.path.join({tmp!r}, "lib.so")
    b.BUILD_DIR = os.path.join({tmp!r}, "_build")
    b.build()
    """)


def _child(tmp, env):
    code = CHILD.format(root=ROOT, tmp=str(tmp))
    return subprocess.Popen([sys.executable, "-c", code], env=env)


def test_concurrent_builds_run_once(tmp_path):
    nvcc = tmp_path / "nvcc"
    nvcc.write_text(FAKE_NVCC)
    nvcc.chmod(nvcc.stat().st_mode | stat.S_IXUSR)
    log = tmp_path / "nvcc.log"
    env = dict(os.environ, NVCC=str(nvcc), FAKE_NVCC_LOG=str(log))
    procs = [_child(tmp_path, env) for _ in range(2)]
    assert [p.wait(timeout=120) for p in procs] == [0, 0]
    calls = log.read_text().split()
    assert len(calls) == len(lib_build.SOURCES) + 1, calls   # one compile per source, one link
    assert os.path.exists(tmp_path / "lib.so")
    # fresh now: a third process does not compile
    assert _child(tmp_path, env).wait(timeout=120) == 0
    assert len(log.read_text().split()) == len(calls)
