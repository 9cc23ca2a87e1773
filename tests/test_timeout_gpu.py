"""A bounded inter-block wait that gives up must end the call with
LSTM_ERR_TIMEOUT in the status word and leave the context usable.  The
failure is made on purpose without faulting anything: one block of the FFMA
forward (backward) recurrence withholds one step's arrivals
(LSTM_B200_DEBUG_SKIP_ARRIVAL), and the wait limit is 20 ms
(LSTM_B200_WAIT_TIMEOUT_NS).  LSTM_B200_REC=simt keeps the float32 case on
the FFMA recurrences, where the hook lives, rather than the tensor-core one.  Each case runs in a fresh process because both
settings are read once per process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("kernel", ["fwd", "bwd"])
def test_withheld_arrival_times_out(kernel, cuda_lib):
    env = dict(os.environ, LSTM_B200_WAIT_TIMEOUT_NS="20000000",
               LSTM_B200_DEBUG_SKIP_ARRIVAL=f"{kernel}:1:2", LSTM_B200_REC="simt")
    r = subprocess.run([sys.executable, os.path.join(HERE, "timeout_check.py"), kernel],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "LSTM_ERR_TIMEOUT" in r.stdout
