"""Bounded-wait failure path of the recurrences, run in a fresh process
(the wait limit and the fault injection are read once per process).

argv[1] = "fwd" or "bwd".  The environment sets LSTM_B200_WAIT_TIMEOUT_NS (a
few ms) and LSTM_B200_DEBUG_SKIP_ARRIVAL="<kernel>:1:2": block 1 of every
recurrent launch of that kernel withholds its step-2 arrivals, so the other
blocks of its group give up at their next counter wait -- where no copy is in
flight -- and the call must end with LSTM_ERR_TIMEOUT in the status word,
while the stream and the context stay usable.  Exit code 0 on success."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from layer_lstm_b200 import binding  # noqa: E402
from layer_lstm_b200.runner import DeviceProblem  # noqa: E402
from layer_lstm_b200.workloads import Workload, make_inputs  # noqa: E402


def main():
    which = sys.argv[1]
    wl = Workload("to", L=1, D=1, I=32, H=256, T=8, B=8, dtype="f32", train=which == "bwd", seed=611)
    p = DeviceProblem(make_inputs(wl))
    binding.lstm_timing_reset()
    binding.lstm_timing_enable(True)
    binding.check(p.forward(), "lstm_forward")
    if which == "bwd":
        binding.check(p.backward(), "lstm_backward")
    st = p.status()
    binding.lstm_timing_enable(False)
    print("status", binding.status_string(st))
    # the recurrent kernels that ran (the engine under test)
    print("kernels", " ".join(k for k, (n, _) in binding.lstm_timing_read().items() if n > 0 and "_rec_" in k))
    # the context is still usable: a plain torch computation and a sync
    v = float(torch.arange(10, device="cuda", dtype=torch.float32).sum().item())
    torch.cuda.synchronize()
    ok = st == binding.LSTM_ERR_TIMEOUT and v == 45.0
    sys.exit(0 if ok else 1)


if __name__ == "__main__":
    main()
