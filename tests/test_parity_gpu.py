"""GPU parity: the CUDA library, called through its C ABI, against the CPU
oracle on identical seeded inputs.

Tolerances: float32 path max-abs 1e-5 on out, h_n, c_n and per-tensor
max-rel 1e-4 on gradients (max|g - o| / max|o|); bf16 path max-abs 2e-2 on
outputs and per-tensor max-rel 1e-2 on gradients.  The bf16 gradient bound is
derived from the rounding the bf16 path applies and the oracle does not:
h_t is rounded to bf16 every step of the forward (relative error up to
2^-9 ~ 2e-3 per step, which the backward's saved sequence inherits) and dx,
dh0 are returned in bf16 (another 2^-9); 1e-2 is five bf16 half-ulps.

Small cases cover several tiles and ragged tails of every partition (units,
batch groups, K slices) and the degenerate cases; the five workloads run at
full size in the launch configuration the benchmark times, checked on sampled
batch rows (rows are independent, so the oracle computes a row subset).
"""
import numpy as np
import pytest
import torch

import oracle
from layer_lstm_b200.workloads import WORKLOADS, Workload, bf16_round, make_inputs, select_rows

pytestmark = pytest.mark.gpu

ATOL_F32 = 1e-5
RTOL_GRAD = 1e-4
ATOL_BF16 = 2e-2
RTOL_GRAD_BF16 = 1e-2


def _run_gpu(inp, cuda_lib):
    from layer_lstm_b200.runner import DeviceProblem
    p = DeviceProblem(inp)
    p.step()
    st = p.status()
    assert st == 0, cuda_lib.status_string(st)
    return p, p.results()


def _check_fwd(wl, gpu, ref, rows=None):
    atol = ATOL_F32 if wl.dtype == "f32" else ATOL_BF16
    bt = 0 if wl.batch_first else 1
    for k in ("out", "h_n", "c_n"):
        g = gpu[k]
        if rows is not None:
            g = np.take(g, rows, axis=bt if k == "out" else 1)
        err = np.abs(g - ref[k]).max() if g.size else 0.0
        assert err <= atol, f"{k}: max-abs {err:.3e} > {atol}"


def _relerr(g, o):
    if o.size == 0:
        return 0.0
    return np.abs(g - o).max() / max(np.abs(o).max(), 1e-30)


def _check_bwd(wl, gpu, ref, rows=None, weights=True):
    bt = 0 if wl.batch_first else 1
    rtol = RTOL_GRAD if wl.dtype == "f32" else RTOL_GRAD_BF16
    for k in ("dx", "dh0", "dc0"):
        g = gpu[k]
        if rows is not None:
            g = np.take(g, rows, axis=bt if k == "dx" else 1)
        e = _relerr(g, ref[k])
        assert e <= rtol, f"{k}: max-rel {e:.3e}"
    if not weights:
        return
    keys = ["dw_ih", "dw_hh"] + (["db_ih", "db_hh"] if wl.bias else [])
    for k in keys:
        for i, (g, o) in enumerate(zip(gpu[k], ref[k])):
            e = _relerr(g, o)
            assert e <= rtol, f"{k}[{i}]: max-rel {e:.3e}"


SMALL = {
    "c1_full": WORKLOADS["c1"],
    "f32_ragged_2layer": Workload("s", L=2, D=1, I=37, H=70, T=9, B=13, dtype="f32",
                                  state_std=0.3, seed=101),
    "f32_bi_seqfirst": Workload("s", L=2, D=2, I=20, H=33, T=7, B=5, dtype="f32",
                                state_std=0.3, batch_first=False, seed=102),
    "f32_nobias_3layer": Workload("s", L=3, D=1, I=16, H=40, T=6, B=7, dtype="f32",
                                  bias=False, seed=103),
    "f32_wide_batch": Workload("s", L=1, D=1, I=24, H=48, T=5, B=150, dtype="f32",
                               state_std=0.2, seed=104),
    "bf16_bi_2layer": Workload("s", L=2, D=2, I=64, H=96, T=11, B=9, dtype="bf16",
                               state_std=0.3, seed=105),
    "bf16_uni": Workload("s", L=1, D=1, I=50, H=130, T=8, B=70, dtype="bf16", seed=106),
    "B1_T1": Workload("s", L=2, D=2, I=5, H=12, T=1, B=1, dtype="f32", state_std=0.5, seed=107),
    # tensor-core recurrence: W_hh slice fully in tensor memory (H=128), split
    # between shared and tensor memory (H=576), ragged batch groups
    "bf16_tc_h128_bi": Workload("s", L=2, D=2, I=64, H=128, T=9, B=40, dtype="bf16",
                                state_std=0.3, seed=111),
    "bf16_tc_h576": Workload("s", L=1, D=1, I=128, H=576, T=5, B=20, dtype="bf16",
                             state_std=0.3, seed=112),
    "bf16_tc_seqfirst": Workload("s", L=1, D=2, I=64, H=256, T=6, B=130, dtype="bf16",
                                 batch_first=False, seed=113),
    # 256 batch columns per cluster, K chunks streamed through the stage ring
    # (two groups of 245 columns, ragged); the same with a W_hh chunk in
    # shared memory and an odd number of K chunks (H = 1088: 9 and 8 per
    # block of a pair)
    "bf16_tc_split": Workload("s", L=1, D=1, I=64, H=1024, T=3, B=490, dtype="bf16",
                              state_std=0.3, seed=115),
    "bf16_tc_split_wsmem": Workload("s", L=1, D=1, I=64, H=1088, T=3, B=480, dtype="bf16",
                                    state_std=0.3, seed=116),
    "H1": Workload("s", L=1, D=1, I=3, H=1, T=4, B=3, dtype="f32", state_std=0.5, seed=108),
    # float32 tensor-core recurrence (3xTF32, clusters of H/128 = 2 blocks),
    # bidirectional, one group of 40 of 64 columns
    "f32_tc_bi": Workload("s", L=2, D=2, I=48, H=256, T=7, B=40, dtype="f32", state_std=0.3, seed=117),
    # bf16 projection on 256 x 256 tiles (M = B*T >= 1024) with ragged M (1073) and K (72)
    "bf16_gemm256_ragged": Workload("s", L=2, D=1, I=72, H=128, T=29, B=37, dtype="bf16",
                                    state_std=0.3, seed=114),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small(name, cuda_lib):
    wl = SMALL[name]
    inp = make_inputs(wl)
    _, gpu = _run_gpu(inp, cuda_lib)
    _check_fwd(wl, gpu, oracle.run_inputs(inp))


TRAIN = {
    "f32_ragged_2layer": SMALL["f32_ragged_2layer"].replace(train=True),
    "f32_bi_seqfirst": SMALL["f32_bi_seqfirst"].replace(train=True),
    "f32_nobias_3layer": SMALL["f32_nobias_3layer"].replace(train=True),
    "B1_T1": SMALL["B1_T1"].replace(train=True),
    "f32_bi_wide": Workload("s", L=1, D=2, I=33, H=64, T=6, B=40, dtype="f32", state_std=0.2,
                            train=True, seed=110),
    # float32 on the tensor cores end to end (3xTF32 forward and BPTT
    # recurrences; BPTT clusters of H/32 blocks): H = 256 bidirectional with
    # inter-layer dropout (clusters of 8, two batch groups), H = 128 (clusters
    # of 4, a ragged second batch group), H = 512 (clusters of 16)
    "f32_tc_bi": Workload("s", L=2, D=2, I=48, H=256, T=7, B=40, dtype="f32", state_std=0.3, train=True,
                          dropout=0.2, dropout_seed=23, seed=147),
    "f32_tc_h128": Workload("s", L=2, D=1, I=24, H=128, T=9, B=50, dtype="f32", state_std=0.3, train=True,
                            seed=148),
    "f32_tc_h512": Workload("s", L=1, D=1, I=32, H=512, T=5, B=20, dtype="f32", state_std=0.3, train=True,
                            seed=149),
    # bf16 BPTT: the recurrence in float32 on widened copies (W_hh rows resident
    # in bf16); the weight phase in bf16 (dG rounded to bf16) with float32 sums
    "bf16_bi_2layer": Workload("s", L=2, D=2, I=64, H=96, T=11, B=9, dtype="bf16", state_std=0.3,
                               train=True, seed=141),
    "bf16_uni_ragged": Workload("s", L=1, D=1, I=50, H=130, T=8, B=20, dtype="bf16", state_std=0.3,
                                train=True, seed=142),
    "bf16_bi_seqfirst": Workload("s", L=1, D=2, I=64, H=256, T=6, B=40, dtype="bf16",
                                 batch_first=False, train=True, seed=143),
    "bf16_long": Workload("s", L=2, D=1, I=32, H=64, T=64, B=8, dtype="bf16", state_std=0.3,
                          train=True, seed=144),
    # inter-layer dropout (Philox4x64-10 mask; identical decisions on both sides)
    "f32_dropout_3layer": Workload("s", L=3, D=1, I=20, H=40, T=7, B=9, dtype="f32", state_std=0.3,
                                   train=True, dropout=0.3, dropout_seed=77, seed=151),
    "f32_dropout_bi": Workload("s", L=2, D=2, I=16, H=36, T=6, B=10, dtype="f32", state_std=0.3,
                               train=True, dropout=0.5, dropout_seed=2 ** 63 + 5, seed=152),
    "bf16_dropout_varlen": Workload("s", L=2, D=2, I=32, H=64, T=8, B=12, dtype="bf16", state_std=0.3,
                                    train=True, dropout=0.25, dropout_seed=9, varlen=True, seed=153),
    # c3's layer shapes (H = 1024, bidirectional, 2 layers) on a short sequence
    "bf16_c3_shape": Workload("s", L=2, D=2, I=512, H=1024, T=12, B=8, dtype="bf16", w_k=1 / 32,
                              train=True, seed=145),
    # tensor-core forward in training (H = 128) with inter-layer dropout and
    # variable lengths: saved gates are zero and c is carried at padding
    "bf16_tc_dropout_varlen": Workload("s", L=2, D=2, I=32, H=128, T=8, B=12, dtype="bf16",
                                       state_std=0.3, train=True, dropout=0.25, dropout_seed=19,
                                       varlen=True, seed=146),
}


@pytest.mark.parametrize("name", list(TRAIN))
def test_backward_small(name, cuda_lib):
    wl = TRAIN[name]
    inp = make_inputs(wl)
    rng = np.random.default_rng(5)
    LDBH = (wl.L * wl.D, wl.B, wl.H)
    inp.grad_hn = rng.standard_normal(LDBH).astype(np.float32)
    inp.grad_cn = rng.standard_normal(LDBH).astype(np.float32)
    if wl.dtype == "bf16":
        inp.grad_hn = bf16_round(inp.grad_hn)   # the device holds it in bf16
    _, gpu = _run_gpu(inp, cuda_lib)
    ref = oracle.run_inputs(inp, backward=True)
    _check_fwd(wl, gpu, ref)
    _check_bwd(wl, gpu, ref)


def test_empty_sequence(cuda_lib):
    """T = 0: h_n = h0, c_n = c0; the backward passes grad_hn/grad_cn to dh0/dc0."""
    wl = Workload("e", L=2, D=2, I=5, H=8, T=0, B=3, dtype="f32", state_std=0.5, train=True, seed=120)
    inp = make_inputs(wl)
    rng = np.random.default_rng(1)
    inp.grad_hn = rng.standard_normal((4, 3, 8)).astype(np.float32)
    inp.grad_cn = rng.standard_normal((4, 3, 8)).astype(np.float32)
    _, gpu = _run_gpu(inp, cuda_lib)
    np.testing.assert_array_equal(gpu["h_n"], inp.h0)
    np.testing.assert_array_equal(gpu["c_n"], inp.c0)
    np.testing.assert_array_equal(gpu["dh0"], inp.grad_hn)
    np.testing.assert_array_equal(gpu["dc0"], inp.grad_cn)
    for w in gpu["dw_ih"] + gpu["dw_hh"] + gpu["db_ih"]:
        assert not np.any(w)


def test_empty_batch(cuda_lib):
    wl = Workload("e", L=1, D=1, I=5, H=8, T=4, B=0, dtype="f32", seed=121)
    _run_gpu(make_inputs(wl), cuda_lib)


def test_zero_weight_closed_form_gpu(cuda_lib):
    """W = 0 (pulsatrix zero-initialised module): gates are constants of the
    biases and c_t = f^(t+1) c0 + i g (1 - f^(t+1)) / (1 - f)."""
    wl = Workload("z", L=1, D=1, I=16, H=64, T=20, B=8, dtype="f32", state_std=0.5, w_k=1.0, seed=122)
    inp = make_inputs(wl, zero_weights=True)
    _, gpu = _run_gpu(inp, cuda_lib)
    b = inp.b_ih[0].astype(np.float64) + inp.b_hh[0].astype(np.float64)
    H = wl.H
    sig = lambda z: 1 / (1 + np.exp(-z))
    i, f, g, o = sig(b[:H]), sig(b[H:2 * H]), np.tanh(b[2 * H:3 * H]), sig(b[3 * H:])
    c0 = inp.c0[0].astype(np.float64)
    for t in range(wl.T):
        n = t + 1
        c = f ** n * c0 + i * g * (1 - f ** n) / (1 - f)
        assert np.abs(gpu["out"][:, t, :] - o * np.tanh(c)).max() < ATOL_F32


# ------------------------------------------------------------ full-size workloads
SAMPLE_ROWS = {"c2": [0, 17, 38, 63], "c3": [0, 31], "c4": [0, 200, 511], "c5": [0, 29, 63], "c3t": [0, 31]}


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4"])
def test_workload_forward_full_size(name, cuda_lib):
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    _, gpu = _run_gpu(inp, cuda_lib)
    rows = SAMPLE_ROWS.get(name)
    sub = inp if rows is None else select_rows(inp, rows)
    _check_fwd(wl, gpu, oracle.run_inputs(sub), rows)


@pytest.mark.parametrize("name", ["c5", "c3t"])
def test_workload_training_full_size(name, cuda_lib):
    """The training steps at full size (c5 float32; c3t bf16 on c3's shape,
    tensor-core forward and BPTT).  Row-local results (out, h_n, c_n, dx,
    dh0, dc0) are checked on sampled rows; weight gradients sum over all
    rows, so a second run zeroes grad_out outside the sampled rows and is
    checked against the oracle's gradients of those rows alone (rows are
    independent; the sampled rows' inputs are the same in both runs, so one
    oracle run serves both checks)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    rows = SAMPLE_ROWS[name]
    _, gpu = _run_gpu(inp, cuda_lib)
    sub = select_rows(inp, rows)
    ref = oracle.run_inputs(sub, backward=True)
    _check_fwd(wl, gpu, ref, rows)
    _check_bwd(wl, gpu, ref, rows, weights=False)
    masked = make_inputs(wl)
    keep = np.zeros(wl.B, dtype=bool)
    keep[rows] = True
    masked.grad_out = np.where(keep[:, None, None], masked.grad_out, 0.0).astype(np.float32)
    _, gpu2 = _run_gpu(masked, cuda_lib)
    ref2 = ref
    rtol = RTOL_GRAD if wl.dtype == "f32" else RTOL_GRAD_BF16
    for k in ("dw_ih", "dw_hh", "db_ih", "db_hh"):
        for i, (g, o) in enumerate(zip(gpu2[k], ref2[k])):
            e = _relerr(g, o)
            assert e <= rtol, f"{k}[{i}]: max-rel {e:.3e}"


@pytest.mark.parametrize("env", ["LSTM_B200_REC=simt", "LSTM_B200_GEMM=simt"])
def test_cuda_core_engines(env, cuda_lib):
    """Re-runs shapes that normally take the tensor-core kernels with the
    CUDA-core kernels forced (engine choice is read once per process)."""
    import os
    import subprocess
    import sys
    k, v = env.split("=")
    e = dict(os.environ)
    e[k] = v
    script = os.path.join(os.path.dirname(__file__), "engine_check.py")
    r = subprocess.run([sys.executable, script], env=e, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
