"""lstm_forward_noalloc against lstm_forward (GPU, through the C ABI).

lstm_forward_noalloc serves callers that cannot allocate device memory or
hand the library a workspace (for example a plugin inside a host program
that owns all device memory).  It runs the same inference forward on a fixed
scratch array inside the library.  Two calls in a row on different inputs
must each match lstm_forward with a caller-allocated workspace, within the
float32 tolerance the parity tests use; a problem too large for the scratch
must be refused with LSTM_ERR_WORKSPACE.
"""
import numpy as np
import pytest
import torch

from layer_lstm_b200 import binding
from layer_lstm_b200.runner import DeviceProblem
from layer_lstm_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

ATOL_F32 = 1e-5
ATOL_BF16 = 2e-2


def _noalloc(p):
    out = torch.zeros_like(p.out)
    h_n = torch.zeros_like(p.h_n)
    c_n = torch.zeros_like(p.c_n)
    st = binding.lstm_forward_noalloc(p.desc, p.x, p.h0, p.c0, p.w_ih, p.w_hh, p.b_ih, p.b_hh,
                                      out, h_n, c_n)
    torch.cuda.synchronize()
    return st, dict(out=out.double().cpu().numpy(), h_n=h_n.double().cpu().numpy(),
                    c_n=c_n.double().cpu().numpy())


def test_noalloc_matches_workspace_forward_twice(cuda_lib):
    wl = Workload("na", L=2, D=2, I=64, H=128, T=24, B=12, dtype="f32", state_std=0.3, seed=900)
    for seed in (901, 902):   # two calls in a row; the scratch keeps the previous contents
        inp = make_inputs(wl, seed=seed)
        p = DeviceProblem(inp, train=False)
        binding.check(p.forward(), "lstm_forward")
        ref = p.results()
        st, got = _noalloc(p)
        assert st == binding.LSTM_OK, binding.status_string(st)
        assert binding.lstm_noalloc_query_status() == binding.LSTM_OK
        for k in ("out", "h_n", "c_n"):
            err = np.abs(got[k] - ref[k]).max()
            assert err <= ATOL_F32, f"{k}: {err:.3e}"


def test_noalloc_bf16_tensor_core_plan_twice(cuda_lib):
    """The bf16 inference forward on a shape that takes the tensor-core
    recurrence (its scratch prefix ends at other buffers than the float32
    plan's): two calls in a row against lstm_forward, and the status word of
    each call read back through lstm_noalloc_query_status."""
    wl = Workload("nab", L=1, D=2, I=64, H=128, T=10, B=40, dtype="bf16", state_std=0.3, seed=904)
    for seed in (905, 906):
        inp = make_inputs(wl, seed=seed)
        p = DeviceProblem(inp, train=False)
        binding.check(p.forward(), "lstm_forward")
        ref = p.results()
        st, got = _noalloc(p)
        assert st == binding.LSTM_OK, binding.status_string(st)
        assert binding.lstm_noalloc_query_status() == binding.LSTM_OK
        for k in ("out", "h_n", "c_n"):
            err = np.abs(got[k] - ref[k]).max()
            assert err <= ATOL_BF16, f"{k}: {err:.3e}"


def test_noalloc_rejects_problem_larger_than_scratch(cuda_lib):
    wl = Workload("big", L=1, D=1, I=256, H=512, T=128, B=64, dtype="f32", seed=903)
    p = DeviceProblem(make_inputs(wl), train=False)
    st, _ = _noalloc(p)
    assert st == binding.LSTM_ERR_WORKSPACE
