#!/usr/bin/env python
"""LSTM forward (+ BPTT) throughput on B200 through the C-ABI library.

One step is one pass of the whole hot path over one batch of synthetic input:
the input projection, the persistent recurrence of every layer, and (for the
training workload, the default) the BPTT recurrence, the weight-gradient and
input-gradient GEMMs, plus a gradient all-reduce when N > 1.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

Prints one JSON line (rank 0).  `value` is whole-job sequence tokens/s
(batch x seq_len per step, summed over ranks) with inputs resident on the
device; `e2e` is the same metric with the inputs copied from pinned host
memory and the results read back every step.  L2 is flushed (a 256 MiB write)
between timed steps, outside the timed events.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from layer_lstm_b200.workloads import DESCRIPTIONS, WORKLOADS, make_inputs, select_rows  # noqa: E402

FFMA_LANES_PER_SM = 128
SM_COUNT = 148
SM_MAX_MHZ = 1965.0
TF32_OVER_BF16 = 1.1 / 2.25   # nominal dense tf32 / bf16 ratio


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="c5")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload lines (the other configurations and the bf16 training step on c3's shape) added beside the headline")
    ap.add_argument("--rank-probe", action="store_true", help=argparse.SUPPRESS)
    return ap.parse_args()


def relaunch_as_ranks(n):
    """--gpus N > 1 without a launcher environment: start N ranks of this
    script with torch.distributed.run on this node (127.0.0.1), one per GPU,
    and return their exit status."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.run(cmd).returncode


def _io_tensors(wl, prob):
    """(inputs a user copies in per step, results read back per step)."""
    h_in = {"x": prob.x, "h0": prob.h0, "c0": prob.c0}
    if wl.train:
        h_in["grad_out"] = prob.grad_out
    h_in = {k: v for k, v in h_in.items() if v is not None}
    outs = [prob.out, prob.h_n, prob.c_n]
    if wl.train:
        outs += [prob.dx, prob.dh0, prob.dc0] + prob.dw_ih + prob.dw_hh + \
            (prob.db_ih + prob.db_hh if wl.bias else [])
    return h_in, outs


def measure_e2e(args, wl, inp, prob, step, flush, stream, rank, world, local):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory and reads its results back.  One GPU:
    two problem instances alternate, so step i+1's input copy and step i's
    result copy (copy streams) overlap step i+1's / step i's compute; the time
    is the device span of all steps (L2 flushes included).  Several ranks: the
    copies and the step run back to back on the compute stream, timed per
    step, max over ranks."""
    import torch
    import torch.distributed as dist
    from layer_lstm_b200 import binding
    from layer_lstm_b200.runner import DeviceProblem
    h_in, outs = _io_tensors(wl, prob)
    host_in = {k: v.detach().cpu().pin_memory() for k, v in h_in.items()}
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(o.numel() * o.element_size() for o in outs)
    tokens = wl.B * wl.T * world * args.steps
    if world > 1:
        host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]

        def e2e_step():
            for k, v in host_in.items():
                h_in[k].copy_(v, non_blocking=True)
            step()
            for ho, o in zip(host_out, outs):
                ho.copy_(o, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        dist.barrier()
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            e2e_step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        t = torch.tensor([sum(a.elapsed_time(b) for a, b in ev)], device=prob.x.device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return {"value": tokens / (float(t.item()) / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "overlap": False}

    probs = [prob, DeviceProblem(inp, device=f"cuda:{local}")]
    io = [_io_tensors(wl, p) for p in probs]
    host_out = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs] for _ in probs]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def pipeline(n, t0=None, t1=None):
        in_done = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        out_done = [torch.cuda.Event() for _ in range(n)]
        gate = torch.cuda.Event()
        if t0 is not None:
            t0.record(stream)
        gate.record(stream)

        def copy_in(i):
            with torch.cuda.stream(s_in):
                s_in.wait_event(gate if i < 2 else comp_done[i - 2])   # after the start / its buffers' last reader
                for name, v in host_in.items():
                    io[i % 2][0][name].copy_(v, non_blocking=True)
                in_done[i].record(s_in)

        copy_in(0)
        for i in range(n):
            k = i % 2
            if i + 1 < n:
                copy_in(i + 1)
            flush.zero_()
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])   # results last written to these buffers are read
            probs[k].step(stream)
            comp_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                for ho, o in zip(host_out[k], io[k][1]):
                    ho.copy_(o, non_blocking=True)
                out_done[i].record(s_out)
        for i in range(max(0, n - 2), n):
            stream.wait_event(out_done[i])
        if t1 is not None:
            t1.record(stream)

    pipeline(2)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipeline(args.steps, t0, t1)
    torch.cuda.synchronize()
    for p in probs:
        st = p.status(stream)
        if st != binding.LSTM_OK:
            raise binding.LstmError(st, "e2e steps")
    return {"value": tokens / (t0.elapsed_time(t1) / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "overlap": True,
            "mode": "pipelined: two problem instances alternate, so each step's input copy and "
                    "its neighbour's result copy (copy streams) overlap compute; time = device span"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# --------------------------------------------------------------- work model
ENGINE_SUFFIXES = ("_tc", "_ffma", "_simt")


def kind_base(kind):
    """Kernel kind without its engine suffix (fwd_rec_tc -> fwd_rec)."""
    for suf in ENGINE_SUFFIXES:
        if kind.endswith(suf):
            return kind[: -len(suf)]
    return kind


def kernel_work(wl, kind):
    """Algorithmic work of all launches of `kind` in one step: (units, amount).

    Recurrences and GEMMs count 2 flops per multiply-add of the matrix
    products the method defines (elementwise gate math is not counted)."""
    kind = kind_base(kind)
    B, T, H, D, L, G = wl.B, wl.T, wl.H, wl.D, wl.L, 4 * wl.H
    ins = [wl.in_size(k) for k in range(L)]
    if kind == "fwd_rec":
        return "flop", 2.0 * B * T * D * G * H * L
    if kind == "bwd_rec":
        return "flop", 2.0 * B * T * D * G * H * L
    if kind == "proj_gemm":
        return "flop", sum(2.0 * B * T * D * G * i for i in ins)
    if kind == "dw_gemm":
        return "flop", sum(2.0 * B * T * D * G * (i + H) for i in ins)
    if kind == "dx_gemm":
        return "flop", sum(2.0 * B * T * D * G * i for i in ins)
    return None, 0.0


# Bound of each kernel kind, from the engine suffix the library reports:
#   alu:    FP32 FMA on the CUDA cores, 148 SMs x 128 lanes x 2 flop x max SM clock
#   tensor: tcgen05 tensor cores.  bf16 operands: the measured cuBLAS bf16 burst
#           peak.  fp32 operands run as 3xTF32 (three tf32 products per fp32
#           product): the bf16 peak x 1.1/2.25 (nominal tf32/bf16 dense ratio) / 3.
COUNTED_KINDS = ("fwd_rec", "bwd_rec", "proj_gemm", "dw_gemm", "dx_gemm")


def kind_bound(kind):
    if kind_base(kind) not in COUNTED_KINDS:
        return None
    return "tensor" if kind.endswith("_tc") else "alu"


def alu_peak_tflops():
    return SM_COUNT * FFMA_LANES_PER_SM * 2 * SM_MAX_MHZ * 1e6 / 1e12


def traffic_for(kind, wl_name):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (profiles/ncu_traffic.json records the source
    hash); otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kind}@{wl_name}") or d.get(kind)   # one kind can name several kernels
    if not e or e.get("workload") != wl_name:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if sha != e.get("source_sha"):
        return None
    return float(e["bytes_per_launch"])


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="lstm_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ CPU oracle
def cpu_oracle_rate(wl, rows_target=None, min_seconds=10.0):
    """Times the oracle (as it stands) on a bounded sample of batch rows of the
    workload; returns (tokens/s, cores, sample description, seconds)."""
    import oracle
    threads = oracle.num_threads()
    inp = make_inputs(wl)
    nrows = rows_target or min(wl.B, max(1, threads))
    while True:
        sub = select_rows(inp, list(range(nrows)))
        t0 = time.perf_counter()
        oracle.run_inputs(sub, backward=wl.train)
        dt = time.perf_counter() - t0
        if dt >= min_seconds or nrows >= wl.B or rows_target is not None:
            break
        nrows = min(wl.B, nrows * 2)
    cores = min(threads, nrows)
    kind = "forward + BPTT" if wl.train else "forward"
    sample = f"{nrows} of {wl.B} batch rows, full T/L/H, {kind}, float64"
    return nrows * wl.T / dt, cores, sample, dt


def cpu_oracle_single_thread_rate(wl):
    """The oracle on one host thread over one batch row of the workload
    (tokens/s): the single-core figure beside the all-core one."""
    import oracle
    threads = oracle.num_threads()
    sub = select_rows(make_inputs(wl), [0])
    oracle.set_num_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.run_inputs(sub, backward=wl.train)
        dt = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(threads)
    return wl.T / dt


# ------------------------------------------------------------------ arms
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    import oracle
    threads = oracle.num_threads()
    inp = make_inputs(wl)
    nrows = min(wl.B, max(1, threads))
    sub = select_rows(inp, list(range(nrows)))
    for _ in range(args.warmup):
        oracle.run_inputs(sub, backward=wl.train)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.run_inputs(sub, backward=wl.train)
    dt = time.perf_counter() - t0
    value = nrows * wl.T * args.steps / dt
    sample = f"{nrows} of {wl.B} batch rows per step, full T/L/H, float64"
    line = {
        "impl": "reference", "metric": "sequence tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(threads, nrows),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, n):
    return {"workload": f"{wl.name}: {DESCRIPTIONS[wl.name]}", "global_batch": wl.B * n,
            "seq_len": wl.T, "layers": wl.L, "hidden": wl.H, "input": wl.I,
            "bidirectional": wl.D == 2, "train": wl.train, "parallelism": f"dp{n}",
            "l2": "flushed between timed steps (256 MiB write)"}


def roofline_of(wl, kern, steps, total_ms, peaks):
    """Roofline object of the kernel kind with the largest share of the timed
    steps: achieved = algorithmic work per launch / average launch time (CUDA
    events recorded by the library around every launch on its stream)."""
    dom = max(((k, v) for k, v in kern.items() if v[0] > 0 and kind_bound(k)),
              key=lambda kv: kv[1][1], default=None)
    if dom is None:
        return None
    kind, (launches, kms) = dom
    unit, work_step = kernel_work(wl, kind)
    per_launch = work_step * steps / launches
    avg_s = kms / launches / 1e3
    bound = kind_bound(kind)
    if bound == "alu":
        peak = alu_peak_tflops()
        peak_note = "derived: 148 SMs x 128 FP32 lanes x 2 flop x 1965 MHz"
    elif wl.dtype == "bf16":
        peak = peaks["bf16_tflops"]
        peak_note = f"{peaks['source']} bf16 burst"
    else:
        peak = peaks["bf16_tflops"] * TF32_OVER_BF16 / 3.0
        peak_note = (f"{peaks['source']} bf16 burst x 1.1/2.25 (tf32) / 3 (3xTF32 products "
                     "per fp32 product)")
    achieved = per_launch / avg_s / 1e12
    return {"bound": bound, "kernel": kind, "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic_for(kind, wl.name),
            "peak_source": peak_note, "launches": launches,
            "avg_launch_ms": kms / launches, "share_of_step": kms / total_ms}


def recurrence_target(wl, kern, steps, peaks, sm_mhz):
    """The recurrence against the bound the method's targets name for it.
    bf16, B >= 256: dense bf16 tensor peak (large-batch recurrence).  bf16,
    small batch: reading every on-chip-resident W_hh element once per step,
    at the aggregate shared-memory rate 148 SMs x 128 B/clk x the SM clock
    observed during the run (small-batch recurrence).  float32: the FP32 FMA
    peak on the CUDA cores, the 3xTF32 tensor peak (bf16 x 1.1/2.25 / 3) on
    the tensor cores."""
    rec = [(k, v) for k, v in kern.items() if kind_base(k) == "fwd_rec" and v[0] > 0]
    if not rec:
        return None
    kind, (launches, kms) = rec[0]
    per_step_s = kms / 1e3 / launches / wl.T     # one step of one layer (all directions)
    flop = 2.0 * wl.B * wl.D * 4 * wl.H * wl.H
    if wl.dtype == "bf16" and wl.B < 256:
        clk = sm_mhz or SM_MAX_MHZ
        peak = SM_COUNT * 128 * clk * 1e6 / 1e9          # GB/s
        bytes_step = wl.D * 4 * wl.H * wl.H * 2
        ach = bytes_step / per_step_s / 1e9
        return {"bound": "smem (W_hh on chip, read once per step)", "kernel": kind,
                "us_per_step": per_step_s * 1e6, "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak, "sm_mhz": clk}
    if wl.dtype == "bf16":
        ach = flop / per_step_s / 1e12
        return {"bound": "tensor", "kernel": kind, "us_per_step": per_step_s * 1e6, "achieved": ach,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"]}
    ach = flop / per_step_s / 1e12
    if kind_bound(kind) == "tensor":
        peak = peaks["bf16_tflops"] * TF32_OVER_BF16 / 3.0
        return {"bound": "tensor", "kernel": kind, "us_per_step": per_step_s * 1e6, "achieved": ach,
                "peak": peak, "unit": "TFLOP/s", "frac": ach / peak}
    return {"bound": "alu", "kernel": kind, "us_per_step": per_step_s * 1e6, "achieved": ach,
            "peak": alu_peak_tflops(), "unit": "TFLOP/s", "frac": ach / alu_peak_tflops()}


def time_steps(step, stream, flush, steps, warmup):
    """(total ms over `steps` timed steps, per-kind kernel timing): CUDA events
    on the launching stream around each step, L2 flushed before each."""
    import torch
    from layer_lstm_b200 import binding
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    binding.lstm_timing_reset()
    binding.lstm_timing_enable(True)
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    binding.lstm_timing_enable(False)
    return sum(a.elapsed_time(b) for a, b in evs), binding.lstm_timing_read()


def measure_workloads(names, steps, warmup, local, flush, peaks, sm_mhz):
    """One line per other workload (the parity-test configurations), timed
    the same way as the headline: tokens/s, ms per step and the roofline of
    the dominant kernel, plus the recurrence against its target bound."""
    import torch
    from layer_lstm_b200 import binding
    from layer_lstm_b200.runner import DeviceProblem
    res = {}
    stream = torch.cuda.current_stream()
    for name in names:
        wl = WORKLOADS[name]
        prob = DeviceProblem(make_inputs(wl), device=f"cuda:{local}")
        total_ms, kern = time_steps(lambda: prob.step(stream), stream, flush, steps, warmup)
        st = prob.status(stream)
        if st != binding.LSTM_OK:
            raise binding.LstmError(st, f"workload {name}")
        res[name] = {
            "workload": DESCRIPTIONS[name], "ms_per_step": total_ms / steps,
            "value": wl.B * wl.T * steps / (total_ms / 1e3), "unit": "tokens/s", "steps": steps,
            "kernels_ms": {k: round(v[1] / steps, 4) for k, v in kern.items() if v[0]},
            "roofline": roofline_of(wl, kern, steps, total_ms, peaks),
            "recurrence": recurrence_target(wl, kern, steps, peaks, sm_mhz),
        }
        del prob
        torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    from layer_lstm_b200 import binding, dp
    from layer_lstm_b200.runner import DeviceProblem

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    binding.load()
    wl = WORKLOADS[args.workload]
    inp = dp.rank_inputs(wl, rank)
    prob = DeviceProblem(inp, device=f"cuda:{local}")
    stream = torch.cuda.current_stream()
    if wl.train:
        bucket = dp.GradBucket.adopt(prob, wl.bias)

        def step():
            dp.train_step(lambda: prob.step(stream), bucket, world)
    else:
        def step():
            prob.step(stream)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=prob.x.device)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = prob.status(stream)
    if st != binding.LSTM_OK:
        raise binding.LstmError(st, "warm-up")

    # ------------------------------------------------ device-resident timing
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    total_ms, kern = time_steps(step, stream, flush, args.steps, 0)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    st = prob.status(stream)
    if st != binding.LSTM_OK:
        raise binding.LstmError(st, "timed steps")
    t = torch.tensor([total_ms], device=prob.x.device, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    tokens = wl.B * wl.T * world * args.steps
    value = tokens / (total_ms / 1e3)

    # ------------------------------------------------------ end to end (host)
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, wl, inp, prob, step, flush, stream, rank, world, local)

    peaks = load_peaks()
    roof = roofline_of(wl, kern, args.steps, total_ms, peaks)
    sm_mhz = clocks.get("sm_mhz") if clocks else None

    # ------------------------------------------ the other workloads (1 GPU)
    others = None
    if rank == 0 and world == 1 and not args.no_workloads:
        names = [n for n in ("c1", "c2", "c3", "c4", "c5", "c3t") if n != wl.name]
        others = measure_workloads(names, steps=10, warmup=3, local=local, flush=flush, peaks=peaks,
                                   sm_mhz=sm_mhz)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample, secs = cpu_oracle_rate(wl)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": sample, "seconds": round(secs, 2),
               "single_thread": {"value": cpu_oracle_single_thread_rate(wl), "unit": "tokens/s",
                                 "cores": 1, "sample": "1 batch row, full T/L/H"}}

    if rank == 0:
        data = "synthetic (seeded)" if world == 1 else \
            "synthetic (seeded; weights shared, each rank its own batch)"
        line = {
            "metric": "sequence tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": data,
            "config": workload_config(wl, world), "e2e": e2e,
            "gpu_launches": int(sum(v[0] for v in kern.values())),
            "kernels_ms": {k: round(v[1] / args.steps, 4) for k, v in kern.items() if v[0]},
            "roofline": roof, "recurrence": recurrence_target(wl, kern, args.steps, peaks, sm_mhz),
            "cpu_baseline": cpu, "clocks": clocks,
            "workloads": others,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_as_ranks(args.gpus))
    world, rank, _ = dist_setup(args)
    if world != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks")
    if args.rank_probe:
        print(f"rank-probe {rank} of {world}", flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
