"""The per-step trace facility (lstm_trace_enable / lstm_trace_read): it
records one row per step for block 0 of the last recurrent launch, with the
events of each step in the order the kernel passes them.  Instrumentation
only; parity of the traced runs is covered elsewhere."""
import numpy as np
import pytest

from layer_lstm_b200 import binding
from layer_lstm_b200.workloads import Workload

CASES = {
    "fwd_ffma": (Workload("t", L=1, D=1, I=16, H=64, T=12, B=8, dtype="f32", seed=131), "fwd",
                 binding.LSTM_TRACE_FWD_REC_FFMA, [0, 1, 2, 3, 4, 5]),
    "bwd_ffma": (Workload("t", L=1, D=1, I=16, H=64, T=12, B=8, dtype="f32", train=True, seed=132), "bwd",
                 binding.LSTM_TRACE_BWD_REC_FFMA, [0, 1, 2, 3, 4, 5]),
    "fwd_tc": (Workload("t", L=1, D=1, I=64, H=256, T=12, B=40, dtype="bf16", seed=133), "fwd",
               binding.LSTM_TRACE_FWD_REC_TC, [0, 9, 3, 4, 5, 6, 7, 8]),
}


def test_trace_read_before_any_trace():
    kind, rows = binding.lstm_trace_read(4)
    assert (kind, rows) == (0, []) or kind in (1, 2, 3)


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_trace_rows(name, cuda_lib, monkeypatch):
    import layer_lstm_b200.trace_steps as ts
    wl, kernel, want_kind, order = CASES[name]
    monkeypatch.setitem(ts.WORKLOADS, "trace_case", wl)
    kind, steps, phases = ts.run("trace_case", kernel)
    assert kind == want_kind
    assert steps == wl.T
    k, rows = binding.lstm_trace_read()
    t = np.array(rows, dtype=np.int64)
    assert t.shape == (wl.T, binding.LSTM_TRACE_EVENTS)
    for s in range(1, wl.T):
        stamps = t[s, order]
        assert np.all(stamps > 0), (s, stamps)
        assert np.all(np.diff(stamps) >= 0), (s, stamps)
    assert all(v >= 0 for v in phases.values())
