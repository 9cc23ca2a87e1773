"""Data-parallel training step on 2 CPU ranks (gloo).

Batch rows are independent in the forward and the backward, so sharding the
batch over ranks and summing the flattened weight/bias gradients with one
all-reduce must reproduce the full-batch gradients, while row-local results
(out, dx, dh0, dc0) stay on their rank.  This is the exchange the benchmark
performs for N > 1 (one all-reduce of the flat gradient buffer per step).
The per-rank gradients come from the CPU oracle, so this runs without a GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from layer_lstm_b200.workloads import Workload, make_inputs, select_rows

WL = Workload("dp", L=2, D=2, I=6, H=5, T=4, B=6, dtype="f32", state_std=0.3, train=True, seed=77)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _flat(r):
    return np.concatenate([a.ravel() for a in r["dw_ih"] + r["dw_hh"] + r["db_ih"]])


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    oracle.set_num_threads(1)
    inp = make_inputs(WL)
    rows = np.array_split(np.arange(WL.B), world)[rank]
    r = oracle.run_inputs(select_rows(inp, rows), backward=True)
    buf = torch.from_numpy(_flat(r))
    dist.all_reduce(buf)
    q.put((rank, buf.numpy(), r["dx"], list(rows)))
    dist.barrier()
    dist.destroy_process_group()


def test_batch_sharded_gradients_allreduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    full = oracle.run_inputs(make_inputs(WL), backward=True)
    want = _flat(full)
    for rank, got, dx, rows in res:
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dx, full["dx"][rows], rtol=0, atol=1e-13)
