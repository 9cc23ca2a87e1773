"""Device buffers for one LSTM problem and the C-ABI calls on them.

Allocation goes through PyTorch (device memory and streams only); every step
of the computation runs in liblstm_b200.so through ``binding``.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding
from .workloads import Inputs, Workload


def torch_dtype(wl: Workload):
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def desc_for(wl: Workload) -> binding.lstm_desc:
    return binding.make_desc(wl.I, wl.H, wl.L, wl.D == 2, wl.bias, wl.batch_first, wl.B, wl.T,
                             binding.LSTM_F32 if wl.dtype == "f32" else binding.LSTM_BF16,
                             wl.dropout, wl.dropout_seed)


class DeviceProblem:
    """Inputs, weights, outputs, workspace and reserve of one problem on a GPU."""

    def __init__(self, inp: Inputs, device="cuda", train: bool | None = None):
        wl = inp.wl
        self.wl = wl
        self.inp = inp
        self.train = wl.train if train is None else train
        dt = torch_dtype(wl)
        self.dt = dt
        self.device = device

        def dev(a, dtype=dt):
            if a is None:
                return None
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=dtype)

        self.desc = desc_for(wl)
        self.lengths = None
        if getattr(inp, "lengths", None) is not None:
            self.lengths = torch.from_numpy(np.ascontiguousarray(inp.lengths, dtype=np.int32)).to(device)
        self.x = dev(inp.x)
        self.h0 = dev(inp.h0)
        self.c0 = dev(inp.c0, torch.float32)
        self.w_ih = [dev(w) for w in inp.w_ih]
        self.w_hh = [dev(w) for w in inp.w_hh]
        self.b_ih = [dev(b) for b in inp.b_ih] if inp.b_ih is not None else None
        self.b_hh = [dev(b) for b in inp.b_hh] if inp.b_hh is not None else None
        LD, B, H, T = wl.L * wl.D, wl.B, wl.H, wl.T
        oshape = (B, T, wl.D * H) if wl.batch_first else (T, B, wl.D * H)
        self.out = torch.zeros(oshape, device=device, dtype=dt)
        self.h_n = torch.zeros((LD, B, H), device=device, dtype=dt)
        self.c_n = torch.zeros((LD, B, H), device=device, dtype=torch.float32)
        ws = binding.lstm_workspace_size(self.desc)
        if ws == 0:
            raise binding.LstmError(binding.LSTM_ERR_INVALID_ARG, "lstm_workspace_size")
        self.workspace = torch.empty(ws, device=device, dtype=torch.uint8)
        self.reserve = None
        if self.train:
            rs = binding.lstm_reserve_size(self.desc)
            self.reserve = torch.empty(max(rs, 256), device=device, dtype=torch.uint8)
            self.grad_out = dev(inp.grad_out)
            self.grad_hn = dev(inp.grad_hn)
            self.grad_cn = dev(inp.grad_cn, torch.float32)
            self.dx = torch.zeros_like(self.x)
            self.dh0 = torch.zeros((LD, B, H), device=device, dtype=dt)
            self.dc0 = torch.zeros((LD, B, H), device=device, dtype=torch.float32)
            self.dw_ih = [torch.zeros(w.shape, device=device, dtype=torch.float32) for w in self.w_ih]
            self.dw_hh = [torch.zeros(w.shape, device=device, dtype=torch.float32) for w in self.w_hh]
            G = 4 * H
            self.db_ih = [torch.zeros(G, device=device, dtype=torch.float32) for _ in range(LD)]
            self.db_hh = [torch.zeros(G, device=device, dtype=torch.float32) for _ in range(LD)]

    def forward(self, stream=None) -> int:
        return binding.lstm_forward(self.desc, self.x, self.h0, self.c0, self.w_ih, self.w_hh,
                                    self.b_ih, self.b_hh, self.out, self.h_n, self.c_n,
                                    self.workspace, self.reserve, stream, lengths=self.lengths)

    def backward(self, stream=None) -> int:
        return binding.lstm_backward(self.desc, self.x, self.h0, self.c0, self.w_ih, self.w_hh,
                                     self.grad_out, self.grad_hn, self.grad_cn, self.reserve,
                                     self.workspace, self.dx, self.dh0, self.dc0, self.dw_ih,
                                     self.dw_hh, self.db_ih if self.wl.bias else None,
                                     self.db_hh if self.wl.bias else None, stream, lengths=self.lengths)

    def step(self, stream=None) -> None:
        binding.check(self.forward(stream), "lstm_forward")
        if self.train:
            binding.check(self.backward(stream), "lstm_backward")

    def status(self, stream=None) -> int:
        return binding.lstm_query_status(self.workspace, stream)

    def results(self) -> dict:
        torch.cuda.synchronize()
        f = lambda t: t.float().cpu().numpy().astype(np.float64)
        r = dict(out=f(self.out), h_n=f(self.h_n), c_n=f(self.c_n))
        if self.train:
            r.update(dx=f(self.dx), dh0=f(self.dh0), dc0=f(self.dc0),
                     dw_ih=[f(t) for t in self.dw_ih], dw_hh=[f(t) for t in self.dw_hh],
                     db_ih=[f(t) for t in self.db_ih] if self.wl.bias else None,
                     db_hh=[f(t) for t in self.db_hh] if self.wl.bias else None)
        return r
