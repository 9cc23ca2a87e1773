"""Per-step timeline of the recurrent kernels (instrumentation).

    python -m layer_lstm_b200.trace_steps --workload c4
    python -m layer_lstm_b200.trace_steps --workload c5 --kernel bwd

Runs the workload once untraced (warm-up), then once with the library's
lstm_trace_enable(1), and prints, for the last recurrent launch of the traced
call, the median over steps of each phase of block 0's step (nanoseconds of
%globaltimer).  --kernel fwd traces the forward (in training mode the
forward is run alone, with its reserve), --kernel bwd the backward.
Synthetic seeded inputs of the named workload; needs a GPU.
"""
import argparse
import json
import sys

import numpy as np
import torch

from layer_lstm_b200 import binding
from layer_lstm_b200.runner import DeviceProblem
from layer_lstm_b200.workloads import WORKLOADS, make_inputs

# phase name -> (event at the end, event at the start, start taken from the previous step)
PHASES = {
    binding.LSTM_TRACE_FWD_REC_FFMA: [
        ("group wait", 1, 0, False),
        ("h tile to shared memory", 2, 1, False),
        ("matvec (first sub-tile)", 3, 2, False),
        ("cell update", 4, 3, False),
        ("publish", 5, 4, False),
        ("step period", 0, 0, True),
    ],
    binding.LSTM_TRACE_BWD_REC_FFMA: [
        ("group wait", 1, 0, False),
        ("partial-dh gather", 2, 1, False),
        ("gate gradients (first sub-tile)", 3, 2, False),
        ("partial-dh products", 4, 3, False),
        ("publish", 5, 4, False),
        ("step period", 0, 0, True),
    ],
    binding.LSTM_TRACE_FWD_REC_TC: [
        ("group wait (after previous publish)", 0, 8, True),
        ("first h chunk lands", 9, 0, False),
        ("MMAs (first chunk to commit)", 3, 9, False),
        ("MMA completion seen", 4, 3, False),
        ("partial sums sent", 5, 4, False),
        ("partner's partial sums received", 6, 5, False),
        ("cell update", 7, 6, False),
        ("h_t out and published", 8, 7, False),
        ("accumulator ready (after previous publish)", 2, 8, True),
        ("Gx loaded (after previous publish)", 10, 8, True),
        ("step period", 8, 8, True),
    ],
    binding.LSTM_TRACE_FWD_REC_TC32: [
        ("group wait (after previous publish)", 0, 8, True),
        ("h tiles land", 9, 0, False),
        ("MMAs issued and committed", 3, 9, False),
        ("MMA completion seen", 4, 3, False),
        ("partial sums sent", 5, 4, False),
        ("owners' partial sums received", 6, 5, False),
        ("cell update", 7, 6, False),
        ("h_t out and published", 8, 7, False),
        ("step period", 8, 8, True),
    ],
    binding.LSTM_TRACE_BWD_REC_TC32: [
        ("group wait (after previous publish)", 0, 8, False),
        ("da tiles land", 9, 0, False),
        ("MMAs issued and committed", 3, 9, False),
        ("MMA completion seen", 4, 3, False),
        ("partial sums sent", 5, 4, False),
        ("owners' partial sums received", 6, 5, False),
        ("gate gradients", 7, 6, False),
        ("published (next row)", 8, 7, True),
        ("step period", 0, 0, True),
    ],
}
KIND_NAMES = {binding.LSTM_TRACE_FWD_REC_FFMA: "fwd_rec_ffma", binding.LSTM_TRACE_BWD_REC_FFMA: "bwd_rec_ffma",
              binding.LSTM_TRACE_FWD_REC_TC: "fwd_rec_tc", binding.LSTM_TRACE_FWD_REC_TC32: "fwd_rec_tc32",
              binding.LSTM_TRACE_BWD_REC_TC32: "bwd_rec_tc32"}


def summarize(kind, rows):
    """{phase: median ns} over the steps where both events were recorded
    (the first and last step are left out: no predecessor / no successor)."""
    t = np.array(rows, dtype=np.int64)
    n = t.shape[0]
    out = {}
    for name, e_end, e_start, prev in PHASES[kind]:
        vals = []
        for s in range(2, n - 1):
            a = t[s - 1, e_start] if prev else t[s, e_start]
            b = t[s, e_end]
            if a > 0 and b > 0:
                vals.append(b - a)
        if vals:
            out[name] = int(np.median(vals))
    return out


def run(workload, kernel):
    wl = WORKLOADS[workload]
    p = DeviceProblem(make_inputs(wl))
    if kernel == "bwd" and not p.train:
        raise SystemExit(f"{workload} is a forward-only workload; no backward to trace")

    def call():
        binding.check(p.forward(), "lstm_forward")
        if kernel == "bwd":
            binding.check(p.backward(), "lstm_backward")

    call()
    torch.cuda.synchronize()
    binding.lstm_trace_enable(True)
    try:
        call()
        torch.cuda.synchronize()
    finally:
        binding.lstm_trace_enable(False)
    st = p.status()
    if st != binding.LSTM_OK:
        raise binding.LstmError(st, "traced call")
    kind, rows = binding.lstm_trace_read()
    if kind == 0 or not rows:
        raise SystemExit("nothing traced")
    return kind, len(rows), summarize(kind, rows)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="c4", choices=sorted(WORKLOADS))
    ap.add_argument("--kernel", default="fwd", choices=["fwd", "bwd"])
    ap.add_argument("--json", action="store_true", help="one JSON line instead of a table")
    args = ap.parse_args(argv)
    kind, steps, phases = run(args.workload, args.kernel)
    if args.json:
        print(json.dumps({"workload": args.workload, "kernel": KIND_NAMES[kind], "steps": steps,
                          "median_ns": phases}))
        return 0
    print(f"{args.workload}: {KIND_NAMES[kind]}, block 0, {steps} steps traced (median over steps 2..T-2, ns)")
    for name, v in phases.items():
        print(f"  {name:45s} {v:8d}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
