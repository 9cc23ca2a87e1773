"""lstm_forward inside a captured CUDA graph: the library enqueues only
stream-ordered work (no host synchronisation), so a capture of one call
replays to the same results as the eager call, bit for bit, for the FFMA
recurrence (float32, cooperative launch) and the tensor-core recurrence
(bf16, cluster launch)."""
import numpy as np
import pytest
import torch

from layer_lstm_b200 import binding
from layer_lstm_b200.runner import DeviceProblem
from layer_lstm_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "f32_ffma": Workload("g", L=2, D=1, I=24, H=48, T=9, B=11, dtype="f32", state_std=0.3, seed=171),
    "bf16_tc": Workload("g", L=1, D=2, I=64, H=256, T=8, B=40, dtype="bf16", state_std=0.3, seed=172),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_graph_replay_matches_eager(name, cuda_lib):
    wl = CASES[name]
    p = DeviceProblem(make_inputs(wl))
    binding.check(p.forward(), "eager forward")
    torch.cuda.synchronize()
    eager = {k: v.clone() for k, v in (("out", p.out), ("h_n", p.h_n), ("c_n", p.c_n))}
    for t in (p.out, p.h_n, p.c_n):
        t.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        st = p.forward(stream=s)
    assert st == binding.LSTM_OK, binding.status_string(st)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert p.status() == binding.LSTM_OK
    for k, v in (("out", p.out), ("h_n", p.h_n), ("c_n", p.c_n)):
        assert torch.equal(v, eager[k]), k
