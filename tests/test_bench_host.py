"""Host-side bookkeeping of the benchmark and the step-timeline tool (CPU).

bench.py turns CUDA-event durations into a roofline fraction: the work model
(flops per step of each kernel kind), the bound chosen from the engine
suffix, and the derived CUDA-core peak must be right for the fraction to
mean anything.  trace_steps.summarize turns raw %globaltimer stamps into
per-phase medians, with phases that start in the previous step.
"""
import numpy as np
import pytest

import bench
from layer_lstm_b200 import trace_steps
from layer_lstm_b200.workloads import WORKLOADS


def _macs_of_products(wl):
    """Multiply-adds of the matrix products of one training step, counted by
    building each product's operand shapes (not from the closed formulas)."""
    G = 4 * wl.H
    rows = wl.B * wl.T                       # one row per (batch row, step)
    out = {"proj": 0, "rec": 0, "dw": 0, "dx": 0}
    for k in range(wl.L):
        fan_in = wl.I if k == 0 else wl.D * wl.H
        for _ in range(wl.D):
            a, b = (rows, fan_in), (fan_in, G)          # X . W_ih^T
            out["proj"] += a[0] * a[1] * b[1]
            a, b = (wl.B, wl.H), (wl.H, G)              # h_{t-1} . W_hh^T, every step
            out["rec"] += wl.T * a[0] * a[1] * b[1]
            a, b = (G, rows), (rows, fan_in + wl.H)     # dG^T . [X | H_{-1}]
            out["dw"] += a[0] * a[1] * b[1]
            a, b = (rows, G), (G, fan_in)               # dG . W_ih
            out["dx"] += a[0] * a[1] * b[1]
    return out


@pytest.mark.parametrize("name", ["c2", "c3", "c4", "c5"])
def test_work_model_counts_two_flops_per_multiply_add(name):
    wl = WORKLOADS[name]
    macs = _macs_of_products(wl)
    assert bench.kernel_work(wl, "fwd_rec_ffma") == ("flop", 2.0 * macs["rec"])
    assert bench.kernel_work(wl, "fwd_rec_tc") == ("flop", 2.0 * macs["rec"])
    assert bench.kernel_work(wl, "bwd_rec_ffma") == ("flop", 2.0 * macs["rec"])
    assert bench.kernel_work(wl, "proj_gemm_tc") == ("flop", 2.0 * macs["proj"])
    assert bench.kernel_work(wl, "dw_gemm_tc") == ("flop", 2.0 * macs["dw"])
    assert bench.kernel_work(wl, "dx_gemm_tc") == ("flop", 2.0 * macs["dx"])
    assert bench.kernel_work(wl, "transpose")[0] is None


def test_bound_follows_engine_suffix():
    assert bench.kind_bound("fwd_rec_ffma") == "alu"
    assert bench.kind_bound("bwd_rec_ffma") == "alu"
    assert bench.kind_bound("fwd_rec_tc") == "tensor"
    assert bench.kind_bound("dw_gemm_tc") == "tensor"
    assert bench.kind_bound("proj_gemm_simt") == "alu"
    # bookkeeping kernels are never the roofline object
    for kind in ("pack", "transpose", "db_reduce", "seq_copy", "dropout"):
        assert bench.kind_bound(kind) is None


def test_derived_ffma_peak():
    # 148 SMs x 128 FP32 lanes x 2 flop per FMA x 1965 MHz
    assert bench.alu_peak_tflops() == pytest.approx(74.44992, rel=1e-9)


def test_trace_summary_medians():
    kind = trace_steps.binding.LSTM_TRACE_FWD_REC_FFMA
    n = 8
    rows = np.zeros((n, 16), dtype=np.int64)
    for s in range(n):
        base = 10_000 * (s + 1) + (7 if s % 2 else 0)   # step period 10000 +- 7
        rows[s, 0] = base
        rows[s, 1] = base + 100 + s                      # group wait 100 + s
        rows[s, 2] = rows[s, 1] + 600
        rows[s, 3] = rows[s, 2] + 3000
        rows[s, 4] = rows[s, 3] + 900
        rows[s, 5] = rows[s, 4] + 700
    got = trace_steps.summarize(kind, rows.tolist())
    # medians over steps 2..n-2 (first and last left out)
    assert got["group wait"] == int(np.median([100 + s for s in range(2, n - 1)]))
    assert got["h tile to shared memory"] == 600
    assert got["matvec (first sub-tile)"] == 3000
    assert got["cell update"] == 900
    assert got["publish"] == 700
    periods = [rows[s, 0] - rows[s - 1, 0] for s in range(2, n - 1)]
    assert got["step period"] == int(np.median(periods))


def test_trace_summary_skips_unrecorded_events():
    kind = trace_steps.binding.LSTM_TRACE_FWD_REC_FFMA
    rows = [[0] * 16 for _ in range(6)]
    for s in range(6):
        rows[s][0] = 1000 * (s + 1)
        rows[s][1] = rows[s][0] + 50
    got = trace_steps.summarize(kind, rows)
    assert got["group wait"] == 50
    assert "publish" not in got   # events 4 and 5 never stamped


def test_single_thread_oracle_rate_restores_thread_count():
    import oracle
    before = oracle.num_threads()
    rate = bench.cpu_oracle_single_thread_rate(WORKLOADS["c1"])
    assert rate > 0
    assert oracle.num_threads() == before


def test_recurrence_target_small_batch_is_whh_bytes_per_step():
    """c3 (bf16, B = 32): the target bound is reading the on-chip W_hh of both
    directions once per step at 148 SMs x 128 B/clk."""
    wl = WORKLOADS["c3"]
    steps = 10
    # 10 steps x 2 layers launches, each T = 256 recurrent steps of 2 us
    kern = {"fwd_rec_tc": (steps * wl.L, steps * wl.L * wl.T * 2e-3)}
    r = bench.recurrence_target(wl, kern, steps, bench.load_peaks(), 1965.0)
    assert r["us_per_step"] == pytest.approx(2.0)
    whh_bytes = wl.D * (4 * wl.H) * wl.H * 2
    assert r["achieved"] == pytest.approx(whh_bytes / 2e-6 / 1e9)
    assert r["peak"] == pytest.approx(148 * 128 * 1965e6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])


def test_recurrence_target_large_batch_is_tensor_peak():
    wl = WORKLOADS["c4"]
    kern = {"fwd_rec_tc": (5, 5 * wl.T * 4e-3), "proj_gemm_tc": (5, 1.0)}
    peaks = bench.load_peaks()
    r = bench.recurrence_target(wl, kern, 5, peaks, None)
    flop = 2.0 * wl.B * 4 * wl.H * wl.H
    assert r["bound"] == "tensor"
    assert r["achieved"] == pytest.approx(flop / 4e-6 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / peaks["bf16_tflops"])


def test_recurrence_target_float32_by_engine():
    """c2 (float32): the CUDA-core recurrence against the FP32 FMA peak, the
    tensor-core one against the 3xTF32 peak (bf16 x 1.1/2.25, three products
    per float32 product)."""
    wl = WORKLOADS["c2"]
    peaks = bench.load_peaks()
    flop = 2.0 * wl.B * 4 * wl.H * wl.H
    r = bench.recurrence_target(wl, {"fwd_rec_tc": (4, 4 * wl.T * 5e-3)}, 2, peaks, None)
    assert r["bound"] == "tensor"
    assert r["achieved"] == pytest.approx(flop / 5e-6 / 1e12)
    assert r["peak"] == pytest.approx(peaks["bf16_tflops"] * 1.1 / 2.25 / 3)
    r = bench.recurrence_target(wl, {"fwd_rec_ffma": (4, 4 * wl.T * 5e-3)}, 2, peaks, None)
    assert r["bound"] == "alu"
    assert r["peak"] == pytest.approx(bench.alu_peak_tflops())


def test_roofline_picks_largest_counted_kind():
    wl = WORKLOADS["c5"]
    kern = {"fwd_rec_ffma": (4, 3.0), "bwd_rec_ffma": (4, 4.0), "transpose": (40, 9.0),
            "dw_gemm_tc": (8, 1.0)}
    r = bench.roofline_of(wl, kern, 2, 10.0, bench.load_peaks())
    assert r["kernel"] == "bwd_rec_ffma"
    per_launch = bench.kernel_work(wl, "bwd_rec_ffma")[1] * 2 / 4
    assert r["achieved"] == pytest.approx(per_launch / 1e-3 / 1e12)
    assert r["share_of_step"] == pytest.approx(0.4)
