"""Seeded synthetic inputs for the LSTM workloads.

This module only draws random numbers and rounds them to the storage type; it
holds none of the LSTM arithmetic.  The same arrays feed the CUDA library and
the CPU oracle, so both sides always see identical values.

Shapes follow the warp_nn LSTM API page ("Learnable parameters" table and the
``__call__`` parameter list): weight_ih_l{k} is (4H, in_k) with in_0 = I and
in_k = D*H for k > 0, weight_hh_l{k} is (4H, H), the biases are 4H long, x is
(B, T, I), h0/c0/h_n/c_n are (L*D, B, H) and out is (B, T, D*H).  Parameters are
drawn from U(-k, k); the warp_nn page gives k = 1/sqrt(hidden_size) as its
default, the five workloads below state their own k.

Draw order (one numpy PCG64 stream per workload): x, h0, c0, then for each
(layer, direction) in layer-major order W_ih, W_hh, b_ih, b_hh, then grad_out.
Values are drawn in float64 and rounded once to float32; bf16 workloads then
round x, h0, the weights and the biases to bf16 (round to nearest, ties to
even) while c0 stays float32.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    L: int                 # num_layers
    D: int                 # 1 + bidirectional
    I: int                 # input_size
    H: int                 # hidden_size
    T: int                 # seq_len
    B: int                 # batch
    dtype: str             # "f32" or "bf16": x, W, b, h0, out, h_n storage type
    train: bool = False    # forward + BPTT when true
    state_std: float = 0.0  # h0, c0 ~ N(0, state_std^2); 0 means h0 = c0 = 0
    w_k: float | None = None  # weights and biases ~ U(-w_k, w_k); None -> 1/sqrt(H)
    bias: bool = True
    batch_first: bool = True
    seed: int = 0
    varlen: bool = False   # per-row lengths ~ U{0..T} (drawn last), else all rows length T
    dropout: float = 0.0   # inter-layer dropout probability of the training forward
    dropout_seed: int = 0  # key word 0 of its Philox4x64-10 stream

    @property
    def G(self) -> int:
        return 4 * self.H

    def in_size(self, layer: int) -> int:
        return self.I if layer == 0 else self.D * self.H

    @property
    def k(self) -> float:
        return self.w_k if self.w_k is not None else 1.0 / math.sqrt(self.H)

    def tokens(self) -> int:
        return self.B * self.T

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads, seeds 1000 + index.
WORKLOADS = {
    "c1": Workload("c1", L=1, D=1, I=8, H=16, T=5, B=4, dtype="f32",
                   w_k=0.25, seed=1001),
    "c2": Workload("c2", L=2, D=1, I=256, H=512, T=128, B=64, dtype="f32",
                   state_std=0.1, w_k=1.0 / math.sqrt(512), seed=1002),
    "c3": Workload("c3", L=2, D=2, I=512, H=1024, T=256, B=32, dtype="bf16",
                   w_k=1.0 / 32, seed=1003),
    "c4": Workload("c4", L=1, D=1, I=1024, H=1024, T=64, B=512, dtype="bf16",
                   w_k=1.0 / 32, seed=1004),
    "c5": Workload("c5", L=2, D=1, I=256, H=512, T=128, B=64, dtype="f32",
                   train=True, state_std=0.1, w_k=1.0 / math.sqrt(512), seed=1005),
    # bf16 BPTT on c3's shape (bidirectional, bf16 weights and activations)
    "c3t": Workload("c3t", L=2, D=2, I=512, H=1024, T=256, B=32, dtype="bf16",
                    train=True, w_k=1.0 / 32, seed=1006),
}

DESCRIPTIONS = {
    "c1": "1-layer LSTM I8 H16 T5 B4 fp32 forward",
    "c2": "2-layer LSTM I256 H512 T128 B64 fp32 forward",
    "c3": "2-layer bidirectional LSTM I512 H1024 T256 B32 bf16 forward",
    "c4": "1-layer LSTM I1024 H1024 T64 B512 bf16 forward",
    "c5": "2-layer LSTM I256 H512 T128 B64 fp32 forward + BPTT training step",
    "c3t": "2-layer bidirectional LSTM I512 H1024 T256 B32 bf16 forward + BPTT training step",
}


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even).

    Returns float32 values that are exactly representable in bf16.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The upper 16 bits of bf16-representable float32 values (the bf16 encoding)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass
class Inputs:
    """Host arrays (float32 values; bf16 workloads hold bf16-representable values)."""
    wl: Workload
    x: np.ndarray            # (B, T, I) if batch_first else (T, B, I)
    h0: np.ndarray | None    # (L*D, B, H)
    c0: np.ndarray | None    # (L*D, B, H), always float32
    w_ih: list               # [L*D] of (4H, in_l)
    w_hh: list               # [L*D] of (4H, H)
    b_ih: list | None        # [L*D] of (4H,)
    b_hh: list | None
    grad_out: np.ndarray | None = None   # same layout as out
    grad_hn: np.ndarray | None = None
    grad_cn: np.ndarray | None = None
    lengths: np.ndarray | None = None    # (B,) int32 valid steps per row, or None (all T)


def make_inputs(wl: Workload, seed: int | None = None, zero_weights: bool = False) -> Inputs:
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    L, D, I, H, T, B = wl.L, wl.D, wl.I, wl.H, wl.T, wl.B
    G = 4 * H

    def normal(shape, std=1.0):
        return (rng.standard_normal(size=shape) * std).astype(np.float32)

    def uniform(shape, k):
        return rng.uniform(-k, k, size=shape).astype(np.float32)

    x = normal((B, T, I))
    if wl.state_std > 0.0:
        h0 = normal((L * D, B, H), wl.state_std)
        c0 = normal((L * D, B, H), wl.state_std)
    else:
        h0 = None
        c0 = None
    w_ih, w_hh, b_ih, b_hh = [], [], [], []
    for layer in range(L):
        for _d in range(D):
            w_ih.append(uniform((G, wl.in_size(layer)), wl.k))
            w_hh.append(uniform((G, H), wl.k))
            b_ih.append(uniform((G,), wl.k))
            b_hh.append(uniform((G,), wl.k))
    grad_out = normal((B, T, D * H)) if wl.train else None

    if zero_weights:
        w_ih = [np.zeros_like(w) for w in w_ih]
        w_hh = [np.zeros_like(w) for w in w_hh]
    if not wl.bias:
        b_ih = None
        b_hh = None
    if wl.dtype == "bf16":
        x = bf16_round(x)
        h0 = bf16_round(h0) if h0 is not None else None
        w_ih = [bf16_round(w) for w in w_ih]
        w_hh = [bf16_round(w) for w in w_hh]
        if b_ih is not None:
            b_ih = [bf16_round(b) for b in b_ih]
            b_hh = [bf16_round(b) for b in b_hh]
        if grad_out is not None:
            grad_out = bf16_round(grad_out)   # the device holds it in bf16
    if not wl.batch_first:
        x = np.ascontiguousarray(x.transpose(1, 0, 2))
        if grad_out is not None:
            grad_out = np.ascontiguousarray(grad_out.transpose(1, 0, 2))
    lengths = None
    if wl.varlen:
        # drawn after everything else, so the other arrays match the fixed-length draw;
        # one row always has the full length and one (if B > 1) is empty
        lengths = rng.integers(0, T + 1, size=B).astype(np.int32)
        if B > 0:
            lengths[0] = T
        if B > 1:
            lengths[-1] = 0
    return Inputs(wl, x, h0, c0, w_ih, w_hh, b_ih, b_hh, grad_out, lengths=lengths)


def select_rows(inp: Inputs, rows) -> Inputs:
    """The same problem restricted to a subset of batch rows (rows are independent)."""
    rows = np.asarray(rows)
    wl = inp.wl.replace(B=len(rows))
    bt = 0 if inp.wl.batch_first else 1

    def take_seq(a):
        return None if a is None else np.ascontiguousarray(np.take(a, rows, axis=bt))

    def take_state(a):
        return None if a is None else np.ascontiguousarray(a[:, rows, :])

    return Inputs(wl, take_seq(inp.x), take_state(inp.h0), take_state(inp.c0),
                  inp.w_ih, inp.w_hh, inp.b_ih, inp.b_hh, take_seq(inp.grad_out),
                  take_state(inp.grad_hn), take_state(inp.grad_cn),
                  None if inp.lengths is None else np.ascontiguousarray(inp.lengths[rows]))
