"""CPU oracle for the LSTM forward and BPTT backward (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package; the CUDA library never does.  The arithmetic lives in
``lstm_oracle.c`` (plain C, IEEE double); this module only marshals numpy
arrays through ctypes.  See the header of ``lstm_oracle.c`` for the equations
and the pages they come from.

Parity pins (tests/test_oracle_pins.py): W = 0 closed form, hand-worked single
steps with rational gates, invariants, batch/direction/layer structural
identities, central finite differences of the BPTT, and torch.nn.LSTM (CPU,
float64) as an independent implementation.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build, build_single as _build_single, LIB_PATH, LIB_PATH_SINGLE

_lib = None


def _load():
    global _lib
    if _lib is None:
        _build()
        lib = ctypes.CDLL(LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        dpp = ctypes.POINTER(dp)
        i = ctypes.c_int
        ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_lstm_forward.argtypes = [i, i, i, i, i, i, i, ip, dp, dp, dp, dpp, dpp, dpp, dpp,
                                            dp, dp, dp]
        lib.oracle_lstm_forward.restype = i
        u64 = ctypes.c_uint64
        lib.oracle_lstm_backward.argtypes = [i, i, i, i, i, i, i, ip, ctypes.c_double, u64,
                                             dp, dp, dp, dpp, dpp, dpp, dpp,
                                             dp, dp, dp, dp, dp, dp, dp, dp, dp, dpp, dpp, dpp, dpp]
        lib.oracle_lstm_backward.restype = i
        lib.oracle_num_threads.restype = i
        u64p = ctypes.POINTER(ctypes.c_uint64)
        lib.oracle_philox4x64_10.argtypes = [u64p, u64p, u64p]
        lib.oracle_philox4x64_10.restype = None
        lib.oracle_set_num_threads.argtypes = [i]
        _lib = lib
    return _lib


def philox4x64_10(ctr, key):
    """The oracle's Philox4x64-10 block: 4 counter words, 2 key words -> 4 words."""
    lib = _load()
    c = (ctypes.c_uint64 * 4)(*[int(v) for v in ctr])
    k = (ctypes.c_uint64 * 2)(*[int(v) for v in key])
    o = (ctypes.c_uint64 * 4)()
    lib.oracle_philox4x64_10(c, k, o)
    return [int(v) for v in o]


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _lengths(lengths, B):
    """(keep-alive array, pointer) for per-row lengths; NULL when None."""
    if lengths is None:
        return None, ctypes.POINTER(ctypes.c_int)()
    a = np.ascontiguousarray(lengths, dtype=np.int32)
    if a.shape != (B,):
        raise ValueError(f"lengths must have shape ({B},)")
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def _ptr_array(arrs):
    dp = ctypes.POINTER(ctypes.c_double)
    if arrs is None:
        return ctypes.POINTER(dp)()
    return (dp * len(arrs))(*[_ptr(a) for a in arrs])


def _dims(x, h_sz, L, D, batch_first):
    if batch_first:
        B, T, I = x.shape
    else:
        T, B, I = x.shape
    return B, T, I


def lstm_forward(x, w_ih, w_hh, b_ih=None, b_hh=None, h0=None, c0=None,
                 num_layers=1, bidirectional=False, batch_first=True, lengths=None):
    """Returns (out, h_n, c_n) as float64 arrays in the same layout as x.
    lengths: per-row valid steps (variable-length batch) or None."""
    lib = _load()
    L, D = int(num_layers), 2 if bidirectional else 1
    x = _f64(x)
    if not batch_first:
        x = np.ascontiguousarray(x.transpose(1, 0, 2))
    B, T, I = x.shape
    H = np.asarray(w_hh[0]).shape[1]
    bias = b_ih is not None
    w_ih = [_f64(w) for w in w_ih]
    w_hh = [_f64(w) for w in w_hh]
    b_ih = [_f64(b) for b in b_ih] if bias else None
    b_hh = [_f64(b) for b in b_hh] if bias else None
    h0, c0 = _f64(h0), _f64(c0)
    out = np.zeros((B, T, D * H))
    h_n = np.zeros((L * D, B, H))
    c_n = np.zeros((L * D, B, H))
    keep, lp = _lengths(lengths, B)
    rc = lib.oracle_lstm_forward(L, D, I, H, B, T, int(bias), lp, _ptr(x), _ptr(h0), _ptr(c0),
                                 _ptr_array(w_ih), _ptr_array(w_hh), _ptr_array(b_ih),
                                 _ptr_array(b_hh), _ptr(out), _ptr(h_n), _ptr(c_n))
    if rc != 0:
        raise RuntimeError(f"oracle_lstm_forward failed with code {rc}")
    if not batch_first:
        out = np.ascontiguousarray(out.transpose(1, 0, 2))
    return out, h_n, c_n


def lstm_backward(x, w_ih, w_hh, grad_out, b_ih=None, b_hh=None, h0=None, c0=None,
                  grad_hn=None, grad_cn=None, num_layers=1, bidirectional=False,
                  batch_first=True, lengths=None, dropout=0.0, dropout_seed=0):
    """Forward + BPTT.  Returns a dict with out, h_n, c_n, dx, dh0, dc0 and the
    per-(layer, direction) lists dw_ih, dw_hh, db_ih, db_hh (float64)."""
    lib = _load()
    L, D = int(num_layers), 2 if bidirectional else 1
    x = _f64(x)
    grad_out = _f64(grad_out)
    if not batch_first:
        x = np.ascontiguousarray(x.transpose(1, 0, 2))
        grad_out = np.ascontiguousarray(grad_out.transpose(1, 0, 2))
    B, T, I = x.shape
    H = np.asarray(w_hh[0]).shape[1]
    G = 4 * H
    bias = b_ih is not None
    w_ih = [_f64(w) for w in w_ih]
    w_hh = [_f64(w) for w in w_hh]
    b_ih = [_f64(b) for b in b_ih] if bias else None
    b_hh = [_f64(b) for b in b_hh] if bias else None
    h0, c0, grad_hn, grad_cn = _f64(h0), _f64(c0), _f64(grad_hn), _f64(grad_cn)
    out = np.zeros((B, T, D * H))
    h_n = np.zeros((L * D, B, H))
    c_n = np.zeros((L * D, B, H))
    dx = np.zeros((B, T, I))
    dh0 = np.zeros((L * D, B, H))
    dc0 = np.zeros((L * D, B, H))
    dw_ih = [np.zeros((G, I if ld // D == 0 else D * H)) for ld in range(L * D)]
    dw_hh = [np.zeros((G, H)) for _ in range(L * D)]
    db_ih = [np.zeros(G) for _ in range(L * D)] if bias else None
    db_hh = [np.zeros(G) for _ in range(L * D)] if bias else None
    keep, lp = _lengths(lengths, B)
    rc = lib.oracle_lstm_backward(L, D, I, H, B, T, int(bias), lp, float(dropout), int(dropout_seed),
                                  _ptr(x), _ptr(h0), _ptr(c0),
                                  _ptr_array(w_ih), _ptr_array(w_hh), _ptr_array(b_ih),
                                  _ptr_array(b_hh), _ptr(grad_out), _ptr(grad_hn), _ptr(grad_cn),
                                  _ptr(out), _ptr(h_n), _ptr(c_n), _ptr(dx), _ptr(dh0), _ptr(dc0),
                                  _ptr_array(dw_ih), _ptr_array(dw_hh), _ptr_array(db_ih),
                                  _ptr_array(db_hh))
    if rc != 0:
        raise RuntimeError(f"oracle_lstm_backward failed with code {rc}")
    if not batch_first:
        out = np.ascontiguousarray(out.transpose(1, 0, 2))
        dx = np.ascontiguousarray(dx.transpose(1, 0, 2))
    return dict(out=out, h_n=h_n, c_n=c_n, dx=dx, dh0=dh0, dc0=dc0,
                dw_ih=dw_ih, dw_hh=dw_hh, db_ih=db_ih, db_hh=db_hh)


_lib_single = None


def lstm_forward_single(x, w_ih, w_hh, b_ih=None, b_hh=None, h0=None, c0=None, num_layers=1,
                        bidirectional=False):
    """The oracle's forward built with every value in float32 (batch-first x);
    returns (out, h_n, c_n) as float32 arrays.  Used only to compare the
    double oracle with a float32 rendition of itself."""
    global _lib_single
    if _lib_single is None:
        _build_single()
        lib = ctypes.CDLL(LIB_PATH_SINGLE)
        fp = ctypes.POINTER(ctypes.c_float)
        fpp = ctypes.POINTER(fp)
        i = ctypes.c_int
        lib.oracle_lstm_forward.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(ctypes.c_int), fp, fp, fp,
                                            fpp, fpp, fpp, fpp, fp, fp, fp]
        lib.oracle_lstm_forward.restype = i
        _lib_single = lib
    fp = ctypes.POINTER(ctypes.c_float)

    def f32(a):
        return None if a is None else np.ascontiguousarray(a, dtype=np.float32)

    def ptr(a):
        return fp() if a is None else a.ctypes.data_as(fp)

    def parr(arrs):
        return ctypes.POINTER(fp)() if arrs is None else (fp * len(arrs))(*[ptr(a) for a in arrs])

    L, D = int(num_layers), 2 if bidirectional else 1
    x = f32(x)
    B, T, I = x.shape
    H = np.asarray(w_hh[0]).shape[1]
    w_ih = [f32(w) for w in w_ih]
    w_hh = [f32(w) for w in w_hh]
    b_ih = [f32(b) for b in b_ih] if b_ih is not None else None
    b_hh = [f32(b) for b in b_hh] if b_hh is not None else None
    h0, c0 = f32(h0), f32(c0)
    out = np.zeros((B, T, D * H), np.float32)
    h_n = np.zeros((L * D, B, H), np.float32)
    c_n = np.zeros((L * D, B, H), np.float32)
    rc = _lib_single.oracle_lstm_forward(L, D, I, H, B, T, int(b_ih is not None), ctypes.POINTER(ctypes.c_int)(),
                                         ptr(x), ptr(h0), ptr(c0), parr(w_ih), parr(w_hh), parr(b_ih),
                                         parr(b_hh), ptr(out), ptr(h_n), ptr(c_n))
    if rc != 0:
        raise RuntimeError(f"oracle_lstm_forward (single) failed with code {rc}")
    return out, h_n, c_n


def run_inputs(inp, backward=False):
    """Run the oracle on a layer_lstm_b200.workloads.Inputs bundle."""
    wl = inp.wl
    kw = dict(b_ih=inp.b_ih, b_hh=inp.b_hh, h0=inp.h0, c0=inp.c0, num_layers=wl.L,
              bidirectional=wl.D == 2, batch_first=wl.batch_first,
              lengths=getattr(inp, "lengths", None))
    if backward:
        return lstm_backward(inp.x, inp.w_ih, inp.w_hh, inp.grad_out, grad_hn=inp.grad_hn,
                             # the library's descriptor holds the probability as a float32
                             grad_cn=inp.grad_cn, dropout=float(np.float32(getattr(wl, "dropout", 0.0))),
                             dropout_seed=getattr(wl, "dropout_seed", 0), **kw)
    out, h_n, c_n = lstm_forward(inp.x, inp.w_ih, inp.w_hh, **kw)
    return dict(out=out, h_n=h_n, c_n=c_n)
