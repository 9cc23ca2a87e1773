"""Parity of the layer wavefront (LSTM_B200_WAVEFRONT=1, chunk length from
LSTM_B200_WAVEFRONT_CHUNK) against the oracle, in a fresh process (both
settings are read once per process).  argv: L I H T B dtype train seed
[rows] -- rows > 0 checks that many sampled batch rows of a full-size
problem.  Exit code 0 when every compared tensor is inside the tolerance of
its dtype."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from layer_lstm_b200.runner import DeviceProblem  # noqa: E402
from layer_lstm_b200.workloads import Workload, make_inputs, select_rows  # noqa: E402


def main():
    L, I, H, T, B = (int(v) for v in sys.argv[1:6])
    dtype, train, seed = sys.argv[6], sys.argv[7] == "1", int(sys.argv[8])
    nrows = int(sys.argv[9]) if len(sys.argv) > 9 else 0
    wl = Workload("wf", L=L, D=1, I=I, H=H, T=T, B=B, dtype=dtype, state_std=0.3, train=train, seed=seed,
                  w_k=None if dtype == "f32" else 1.0 / 32)
    inp = make_inputs(wl)
    p = DeviceProblem(inp)
    p.step()
    if p.status() != 0:
        print("status", p.status())
        sys.exit(2)
    g = p.results()
    rows = list(range(B)) if nrows == 0 else sorted(set(np.linspace(0, B - 1, nrows).astype(int).tolist()))
    ref = oracle.run_inputs(select_rows(inp, rows), backward=train)
    atol = 1e-5 if dtype == "f32" else 2e-2
    rtol = 1e-4 if dtype == "f32" else 1e-2
    bad = 0
    for k in ("out", "h_n", "c_n"):
        a = np.take(g[k], rows, axis=0 if k == "out" else 1)
        err = float(np.abs(a - ref[k]).max())
        print(k, err)
        bad += err > atol
    if train:
        for k in ("dx", "dh0", "dc0"):
            a = np.take(g[k], rows, axis=0 if k == "dx" else 1)
            err = float(np.abs(a - ref[k]).max() / np.abs(ref[k]).max())
            print(k, err)
            bad += err > rtol
        if nrows == 0:
            for k in ("dw_ih", "dw_hh", "db_ih"):
                for a, b in zip(g[k], ref[k]):
                    err = float(np.abs(a - b).max() / np.abs(b).max())
                    print(k, err)
                    bad += err > rtol
    sys.exit(1 if bad else 0)


if __name__ == "__main__":
    main()
