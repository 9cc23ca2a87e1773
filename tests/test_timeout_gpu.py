"""A bounded inter-block wait that gives up must end the call with
LSTM_ERR_TIMEOUT in the status word and leave the context usable.  The
failure is made on purpose without faulting anything: one block of the
forward (backward) recurrence withholds one step's arrivals
(LSTM_B200_DEBUG_SKIP_ARRIVAL), and the wait limit is 20 ms
(LSTM_B200_WAIT_TIMEOUT_NS).  The float32 case (H = 256) takes the
tensor-core recurrences (tc_rec32_kernel, tc_bwd32_kernel: the other blocks
give up at their group-counter wait, with no copy or MMA in flight there,
and every role drains and leaves); LSTM_B200_REC=simt takes the FFMA ones.  Each case runs in a fresh process because both
settings are read once per process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("engine", ["simt", "tc"])
@pytest.mark.parametrize("kernel", ["fwd", "bwd"])
def test_withheld_arrival_times_out(kernel, engine, cuda_lib):
    env = dict(os.environ, LSTM_B200_WAIT_TIMEOUT_NS="20000000",
               LSTM_B200_DEBUG_SKIP_ARRIVAL=f"{kernel}:1:2")
    if engine == "simt":
        env["LSTM_B200_REC"] = "simt"
    else:
        env.pop("LSTM_B200_REC", None)
    r = subprocess.run([sys.executable, os.path.join(HERE, "timeout_check.py"), kernel],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "LSTM_ERR_TIMEOUT" in r.stdout
    assert f"{kernel}_rec_{'ffma' if engine == 'simt' else 'tc'}" in r.stdout, r.stdout
