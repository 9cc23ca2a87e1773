"""Parity of a few shapes against the oracle in a fresh process, so that the
engine switches LSTM_B200_REC / LSTM_B200_GEMM (read once per process) can be
exercised by tests/test_parity_gpu.py::test_cuda_core_engines.  Exit code 0
when every case is inside the tolerances."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from layer_lstm_b200.runner import DeviceProblem  # noqa: E402
from layer_lstm_b200.workloads import Workload, make_inputs  # noqa: E402

CASES = [
    Workload("e", L=2, D=2, I=64, H=128, T=7, B=24, dtype="bf16", state_std=0.3, seed=301),
    Workload("e", L=2, D=1, I=64, H=128, T=6, B=16, dtype="f32", state_std=0.3, train=True, seed=302),
]


def main():
    bad = 0
    for wl in CASES:
        inp = make_inputs(wl)
        p = DeviceProblem(inp)
        p.step()
        assert p.status() == 0
        g = p.results()
        ref = oracle.run_inputs(inp, backward=wl.train)
        atol = 1e-5 if wl.dtype == "f32" else 2e-2
        for k in ("out", "h_n", "c_n"):
            err = float(np.abs(g[k] - ref[k]).max())
            print(wl.dtype, k, err)
            bad += err > atol
        if wl.train:
            for k in ("dx", "dh0", "dc0"):
                err = float(np.abs(g[k] - ref[k]).max() / np.abs(ref[k]).max())
                print(k, err)
                bad += err > 1e-4
            for k in ("dw_ih", "dw_hh", "db_ih"):
                for a, b in zip(g[k], ref[k]):
                    err = float(np.abs(a - b).max() / np.abs(b).max())
                    print(k, err)
                    bad += err > 1e-4
    sys.exit(1 if bad else 0)


if __name__ == "__main__":
    main()
