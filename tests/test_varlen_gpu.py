"""GPU parity of variable-length batches (lstm_forward_varlen /
lstm_backward_varlen) against the oracle on the same seeded inputs and
lengths (one full-length row, one empty row, the rest drawn in 0..T).
Tolerances as for fixed-length batches (see test_parity_gpu)."""
import numpy as np
import pytest

import oracle
from layer_lstm_b200.workloads import Workload, bf16_round, make_inputs

from test_parity_gpu import _check_bwd, _check_fwd, _run_gpu

pytestmark = pytest.mark.gpu

FWD = {
    "f32_uni_2layer": Workload("v", L=2, D=1, I=24, H=48, T=9, B=11, dtype="f32", state_std=0.3,
                               varlen=True, seed=161),
    "f32_bi_seqfirst": Workload("v", L=2, D=2, I=20, H=33, T=7, B=6, dtype="f32", state_std=0.3,
                                batch_first=False, varlen=True, seed=162),
    "bf16_ffma_bi": Workload("v", L=2, D=2, I=64, H=96, T=10, B=9, dtype="bf16", state_std=0.3,
                             varlen=True, seed=163),
    "bf16_tc_bi": Workload("v", L=2, D=2, I=64, H=256, T=9, B=40, dtype="bf16", state_std=0.3,
                           varlen=True, seed=164),
    "bf16_tc_seqfirst": Workload("v", L=1, D=2, I=64, H=128, T=8, B=70, dtype="bf16",
                                 batch_first=False, varlen=True, seed=165),
    # float32 tensor-core recurrence (3xTF32): padding holds h and c
    "f32_tc_bi": Workload("v", L=2, D=2, I=40, H=256, T=8, B=36, dtype="f32", state_std=0.3,
                          varlen=True, seed=167),
}

TRAIN = {
    "f32_uni_2layer": FWD["f32_uni_2layer"].replace(train=True),
    "f32_bi_seqfirst": FWD["f32_bi_seqfirst"].replace(train=True),
    "f32_bi_wide": Workload("v", L=1, D=2, I=33, H=64, T=6, B=40, dtype="f32", state_std=0.2,
                            train=True, varlen=True, seed=166),
    "bf16_bi": FWD["bf16_ffma_bi"].replace(train=True),
    "f32_tc_bi": FWD["f32_tc_bi"].replace(train=True),
}


@pytest.mark.parametrize("name", list(FWD))
def test_varlen_forward(name, cuda_lib):
    wl = FWD[name]
    inp = make_inputs(wl)
    assert inp.lengths is not None and inp.lengths.min() == 0 and inp.lengths.max() == wl.T
    _, gpu = _run_gpu(inp, cuda_lib)
    ref = oracle.run_inputs(inp)
    _check_fwd(wl, gpu, ref)
    # padding is exactly zero in the user output
    for b, n in enumerate(inp.lengths):
        pad = gpu["out"][b, n:] if wl.batch_first else gpu["out"][n:, b]
        assert not np.any(pad)


@pytest.mark.parametrize("name", list(TRAIN))
def test_varlen_backward(name, cuda_lib):
    wl = TRAIN[name]
    inp = make_inputs(wl)
    rng = np.random.default_rng(7)
    LDBH = (wl.L * wl.D, wl.B, wl.H)
    inp.grad_hn = rng.standard_normal(LDBH).astype(np.float32)
    inp.grad_cn = rng.standard_normal(LDBH).astype(np.float32)
    if wl.dtype == "bf16":
        inp.grad_hn = bf16_round(inp.grad_hn)
    _, gpu = _run_gpu(inp, cuda_lib)
    ref = oracle.run_inputs(inp, backward=True)
    _check_fwd(wl, gpu, ref)
    _check_bwd(wl, gpu, ref)


@pytest.mark.parametrize("name", ["f32_uni_2layer", "bf16_tc_bi"])
def test_full_lengths_equal_fixed_length(name, cuda_lib):
    """lengths all equal to T take the same arithmetic as the fixed-length
    entry point: identical outputs, bit for bit."""
    wl = FWD[name]
    inp = make_inputs(wl)
    inp.lengths = np.full(wl.B, wl.T, dtype=np.int32)
    _, a = _run_gpu(inp, cuda_lib)
    inp.lengths = None
    _, b = _run_gpu(inp, cuda_lib)
    for k in ("out", "h_n", "c_n"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)
