"""Data-parallel training step on 2 CPU ranks (gloo), through the product's
data-parallel code (layer_lstm_b200.dp) that the benchmark runs for N > 1.

Batch rows are independent in the forward and the backward, so sharding the
batch over ranks and summing the flat gradient bucket with one all-reduce
must reproduce the full-batch gradients, while row-local results (dx) stay
on their rank.  Each rank's shard gradients come from the CPU oracle (no
GPU here); `dp.train_step` writes them into the bucket's views and
all-reduces exactly as in the benchmark.  A second test checks that
`bench.py --gpus 2` without a launcher environment starts two rank
processes itself.
"""
import os
import subprocess
import sys
import tempfile
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from layer_lstm_b200 import dp
from layer_lstm_b200.workloads import Workload, make_inputs, select_rows

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WL = Workload("dp", L=2, D=2, I=6, H=5, T=4, B=7, dtype="f32", state_std=0.3, train=True, seed=77)


def _flat(r):
    return np.concatenate([a.ravel() for a in r["dw_ih"] + r["dw_hh"] + r["db_ih"]])


def _worker(rank, world, rdzv, q):
    import datetime
    # rendezvous through a file: no port that another process could take first
    dist.init_process_group("gloo", init_method=f"file://{rdzv}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle
    oracle.set_num_threads(1)
    inp = make_inputs(WL)
    rows = dp.shard_rows(WL.B, world, rank)
    shard = select_rows(inp, rows)
    # a stand-in problem holding this rank's gradient tensors, as DeviceProblem does
    LD, G, H = WL.L * WL.D, 4 * WL.H, WL.H
    prob = types.SimpleNamespace(
        dw_ih=[torch.full((G, WL.in_size(i // WL.D)), float("nan")) for i in range(LD)],
        dw_hh=[torch.full((G, H), float("nan")) for _ in range(LD)],
        db_ih=[torch.full((G,), float("nan")) for _ in range(LD)],
        db_hh=[torch.full((G,), float("nan")) for _ in range(LD)])
    bucket = dp.GradBucket.adopt(prob, bias=True)
    res = {}

    def step():   # what the library does on a GPU: write this shard's gradients
        r = oracle.run_inputs(shard, backward=True)
        for dst, src in zip(prob.dw_ih + prob.dw_hh + prob.db_ih, r["dw_ih"] + r["dw_hh"] + r["db_ih"]):
            dst.copy_(torch.from_numpy(src))
        res["dx"] = r["dx"]

    dp.train_step(step, bucket, world)
    db_hh = np.concatenate([t.numpy().ravel() for t in prob.db_hh])
    q.put((rank, bucket.flat.numpy().copy(), db_hh, res["dx"], rows))
    dist.barrier()
    dist.destroy_process_group()


def test_batch_sharded_gradients_allreduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    rdzv = os.path.join(tempfile.mkdtemp(prefix="lstm_dp_"), "rdzv")
    procs = [ctx.Process(target=_worker, args=(r, world, rdzv, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    full = oracle.run_inputs(make_inputs(WL), backward=True)
    want = _flat(full)
    assert sorted(r for _, _, _, _, rows in res for r in rows) == list(range(WL.B))
    # the bucket holds float32 (what the library writes): each shard's sum
    # is rounded once to float32 and the all-reduce adds two of them
    tol = 4 * np.finfo(np.float32).eps * np.abs(want).max()
    for rank, got, db_hh, dx, rows in res:
        np.testing.assert_allclose(got, want, rtol=0, atol=tol)
        np.testing.assert_allclose(db_hh, np.concatenate(full["db_hh"]), rtol=0, atol=tol)
        np.testing.assert_allclose(dx, full["dx"][rows], rtol=0, atol=1e-13)


def test_shard_rows_cover_batch():
    for B in (0, 1, 5, 64):
        for world in (1, 2, 3, 8):
            rows = [r for k in range(world) for r in dp.shard_rows(B, world, k)]
            assert rows == list(range(B))


def test_rank_inputs_share_weights():
    wl = WL.replace(B=3)
    a, b = dp.rank_inputs(wl, 0), dp.rank_inputs(wl, 1)
    base = make_inputs(wl)
    np.testing.assert_array_equal(a.x, base.x)
    for wa, wb in zip(a.w_ih + a.w_hh, b.w_ih + b.w_hh):
        np.testing.assert_array_equal(wa, wb)
    assert not np.array_equal(a.x, b.x)


def test_bench_gpus_flag_starts_one_process_per_rank():
    """bench.py --gpus 2, started without WORLD_SIZE, relaunches itself as 2
    ranks (torch.distributed.run, 127.0.0.1); --rank-probe makes each rank
    report itself and exit before touching a GPU."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--rank-probe"],
                       capture_output=True, text=True, timeout=180, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = sorted(l for l in r.stdout.splitlines() if l.startswith("rank-probe"))
    assert lines == ["rank-probe 0 of 2", "rank-probe 1 of 2"], r.stdout
