"""Data-parallel training over batch shards, one process per GPU.

Batch rows never interact in the LSTM (warp_nn "Long Short-Term Memory
(LSTM)" equation block: every row carries its own h and c), so a batch split
over ranks needs a single exchange per training step: the sum of the weight
and bias gradients over the ranks (pulsatrix LSTMModule, backward(): the
gradients are sums over every row and step, so the sum of per-shard sums is
the full-batch gradient).  Rank-local results (out, h_n, c_n, dx, dh0, dc0)
stay where they were computed.

`GradBucket` lays every gradient of one problem out in one flat float32
buffer so that the exchange is one all-reduce; `train_step` runs one step and
that all-reduce.  The benchmark and the two-rank CPU test call the same code.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from .workloads import Inputs, Workload, make_inputs


def shard_rows(batch: int, world: int, rank: int) -> list:
    """Batch rows of `rank` when `batch` rows are split over `world` ranks
    (contiguous, sizes differing by at most one)."""
    return [int(i) for i in np.array_split(np.arange(batch), world)[rank]]


def rank_inputs(wl: Workload, rank: int) -> Inputs:
    """Inputs of one data-parallel replica: the weights every rank shares
    (the workload's own draw) and this rank's batch of data (x, h0, c0,
    grad_out drawn from the workload seed offset by the rank).  Rank 0 gets
    exactly make_inputs(wl)."""
    base = make_inputs(wl)
    if rank == 0:
        return base
    data = make_inputs(wl, seed=wl.seed + 7919 * rank)
    return Inputs(wl=wl, x=data.x, h0=data.h0, c0=data.c0, w_ih=base.w_ih, w_hh=base.w_hh,
                  b_ih=base.b_ih, b_hh=base.b_hh, grad_out=data.grad_out, grad_hn=data.grad_hn,
                  grad_cn=data.grad_cn, lengths=getattr(data, "lengths", None))


class GradBucket:
    """One flat float32 buffer for the gradients dW_ih, dW_hh and db of a
    problem (order: every dW_ih, every dW_hh, every db_ih).

    `adopt(prob)` points the problem's gradient tensors at views of the
    buffer, so that the library writes the gradients straight into it.  db_hh
    equals db_ih (the two biases enter the gates as a sum), so only db_ih is
    exchanged; `finish()` copies the reduced db_ih into db_hh."""

    def __init__(self, tensors, device=None):
        n = sum(int(t.numel()) for t in tensors)
        dev = device if device is not None else (tensors[0].device if tensors else "cpu")
        self.flat = torch.zeros(n, device=dev, dtype=torch.float32)
        self.views = []
        off = 0
        for t in tensors:
            self.views.append(self.flat[off:off + t.numel()].view(t.shape))
            off += t.numel()
        self._db_pairs = []

    @classmethod
    def adopt(cls, prob, bias: bool) -> "GradBucket":
        grads = list(prob.dw_ih) + list(prob.dw_hh) + (list(prob.db_ih) if bias else [])
        b = cls(grads)
        n = len(prob.dw_ih)
        prob.dw_ih = b.views[:n]
        prob.dw_hh = b.views[n:2 * n]
        if bias:
            prob.db_ih = b.views[2 * n:]
            b._db_pairs = list(zip(prob.db_ih, prob.db_hh))
        return b

    def allreduce(self, group=None) -> None:
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)

    def finish(self) -> None:
        for src, dst in self._db_pairs:
            dst.copy_(src)


def train_step(step, bucket: GradBucket, world: int, group=None) -> None:
    """One data-parallel training step: `step()` computes this rank's
    gradients into the bucket, then (world > 1) one all-reduce sums them."""
    step()
    if world > 1:
        bucket.allreduce(group)
    bucket.finish()
