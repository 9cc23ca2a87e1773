"""Thin ctypes binding of liblstm_b200.so (include/lstm.h).

Argument marshalling only: tensors become device pointers, lists of tensors
become host arrays of device pointers, and every function returns the C
status code.  All computation happens in the CUDA library; there is no other
code path.  PyTorch is used by callers for device memory and streams.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

LSTM_OK = 0
LSTM_ERR_INVALID_ARG = 1
LSTM_ERR_UNSUPPORTED = 2
LSTM_ERR_WORKSPACE = 3
LSTM_ERR_CUDA = 4
LSTM_ERR_TIMEOUT = 5
LSTM_F32 = 0
LSTM_BF16 = 1

EXPORTED = ("lstm_workspace_size", "lstm_reserve_size", "lstm_forward", "lstm_backward",
            "lstm_query_status", "lstm_status_string", "lstm_timing_enable", "lstm_timing_read",
            "lstm_timing_reset", "lstm_forward_noalloc", "lstm_trace_enable", "lstm_trace_read",
            "lstm_forward_varlen", "lstm_backward_varlen", "lstm_noalloc_query_status")
LSTM_NOALLOC_SCRATCH_BYTES = 32 << 20
LSTM_TRACE_MAX_STEPS = 512
LSTM_TRACE_EVENTS = 16
LSTM_TRACE_FWD_REC_FFMA = 1
LSTM_TRACE_BWD_REC_FFMA = 2
LSTM_TRACE_FWD_REC_TC = 3
LSTM_TRACE_FWD_REC_TC32 = 4
LSTM_TRACE_BWD_REC_TC32 = 5


class lstm_kernel_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_longlong),
                ("total_ms", ctypes.c_double)]


class lstm_desc(ctypes.Structure):
    _fields_ = [("input_size", ctypes.c_int), ("hidden_size", ctypes.c_int),
                ("num_layers", ctypes.c_int), ("bidirectional", ctypes.c_int),
                ("bias", ctypes.c_int), ("batch_first", ctypes.c_int),
                ("batch", ctypes.c_int), ("seq_len", ctypes.c_int), ("dtype", ctypes.c_int),
                ("dropout", ctypes.c_float), ("dropout_seed", ctypes.c_ulonglong)]


def make_desc(input_size, hidden_size, num_layers=1, bidirectional=False, bias=True,
              batch_first=True, batch=1, seq_len=1, dtype=LSTM_F32, dropout=0.0,
              dropout_seed=0) -> lstm_desc:
    return lstm_desc(int(input_size), int(hidden_size), int(num_layers), int(bool(bidirectional)),
                     int(bool(bias)), int(bool(batch_first)), int(batch), int(seq_len), int(dtype),
                     float(dropout), int(dropout_seed))


_lib = None


class LstmError(RuntimeError):
    def __init__(self, status, where=""):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


def lib_path() -> str:
    return _build.LIB_PATH


def load(build_if_stale: bool = True):
    """Loads the CUDA library (building it in-tree when sources are newer).

    Raises if the library cannot be built or loaded: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_stale:
        _build.build()
    if not os.path.exists(_build.LIB_PATH):
        raise RuntimeError(f"CUDA library missing: {_build.LIB_PATH}")
    lib = ctypes.CDLL(_build.LIB_PATH)
    vp = ctypes.c_void_p
    vpp = ctypes.POINTER(ctypes.c_void_p)
    dp = ctypes.POINTER(lstm_desc)
    sz = ctypes.c_size_t
    lib.lstm_workspace_size.argtypes = [dp]
    lib.lstm_workspace_size.restype = sz
    lib.lstm_reserve_size.argtypes = [dp]
    lib.lstm_reserve_size.restype = sz
    lib.lstm_forward.argtypes = [dp, vp, vp, vp, vpp, vpp, vpp, vpp, vp, vp, vp, vp, sz, vp, sz, vp]
    lib.lstm_forward.restype = ctypes.c_int
    lib.lstm_backward.argtypes = [dp, vp, vp, vp, vpp, vpp, vp, vp, vp, vp, sz, vp, sz, vp, vp, vp,
                                  vpp, vpp, vpp, vpp, vp]
    lib.lstm_backward.restype = ctypes.c_int
    lib.lstm_forward_varlen.argtypes = [dp, vp] + list(lib.lstm_forward.argtypes[1:])
    lib.lstm_forward_varlen.restype = ctypes.c_int
    lib.lstm_backward_varlen.argtypes = [dp, vp] + list(lib.lstm_backward.argtypes[1:])
    lib.lstm_backward_varlen.restype = ctypes.c_int
    lib.lstm_query_status.argtypes = [vp, vp]
    lib.lstm_query_status.restype = ctypes.c_int
    lib.lstm_status_string.argtypes = [ctypes.c_int]
    lib.lstm_status_string.restype = ctypes.c_char_p
    lib.lstm_timing_enable.argtypes = [ctypes.c_int]
    lib.lstm_timing_enable.restype = ctypes.c_int
    lib.lstm_timing_read.argtypes = [ctypes.POINTER(lstm_kernel_time), ctypes.c_int]
    lib.lstm_timing_read.restype = ctypes.c_int
    lib.lstm_timing_reset.argtypes = []
    lib.lstm_timing_reset.restype = None
    lib.lstm_forward_noalloc.argtypes = [dp, vp, vp, vp, vpp, vpp, vpp, vpp, vp, vp, vp, vp]
    lib.lstm_forward_noalloc.restype = ctypes.c_int
    lib.lstm_noalloc_query_status.argtypes = [vp]
    lib.lstm_noalloc_query_status.restype = ctypes.c_int
    lib.lstm_trace_enable.argtypes = [ctypes.c_int]
    lib.lstm_trace_enable.restype = ctypes.c_int
    lib.lstm_trace_read.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
    lib.lstm_trace_read.restype = ctypes.c_int
    _lib = lib
    return lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _nbytes(t):
    if t is None:
        return 0
    return t.numel() * t.element_size()


def _parr(ts):
    if ts is None:
        return None
    return (ctypes.c_void_p * len(ts))(*[_p(t) for t in ts])


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def status_string(status: int) -> str:
    return load().lstm_status_string(int(status)).decode()


def lstm_status_string(status: int) -> str:
    return status_string(status)


def lstm_workspace_size(desc: lstm_desc) -> int:
    return int(load().lstm_workspace_size(ctypes.byref(desc)))


def lstm_reserve_size(desc: lstm_desc) -> int:
    return int(load().lstm_reserve_size(ctypes.byref(desc)))


def lstm_forward(desc, x, h0, c0, w_ih, w_hh, b_ih, b_hh, out, h_n, c_n, workspace,
                 reserve=None, stream=None, ws_bytes=None, rs_bytes=None, lengths=None) -> int:
    """lengths: device int32 tensor of per-row valid steps (lstm_forward_varlen),
    or None (lstm_forward)."""
    lib = load()
    args = (_p(x), _p(h0), _p(c0), _parr(w_ih), _parr(w_hh),
            _parr(b_ih), _parr(b_hh), _p(out), _p(h_n), _p(c_n),
            _p(workspace), _nbytes(workspace) if ws_bytes is None else ws_bytes,
            _p(reserve), _nbytes(reserve) if rs_bytes is None else rs_bytes,
            _stream(stream))
    if lengths is None:
        return lib.lstm_forward(ctypes.byref(desc), *args)
    return lib.lstm_forward_varlen(ctypes.byref(desc), _p(lengths), *args)


def lstm_backward(desc, x, h0, c0, w_ih, w_hh, grad_out, grad_hn, grad_cn, reserve, workspace,
                  dx, dh0, dc0, dw_ih, dw_hh, db_ih, db_hh, stream=None,
                  ws_bytes=None, rs_bytes=None, lengths=None) -> int:
    lib = load()
    args = (_p(x), _p(h0), _p(c0), _parr(w_ih), _parr(w_hh),
            _p(grad_out), _p(grad_hn), _p(grad_cn), _p(reserve),
            _nbytes(reserve) if rs_bytes is None else rs_bytes,
            _p(workspace), _nbytes(workspace) if ws_bytes is None else ws_bytes,
            _p(dx), _p(dh0), _p(dc0), _parr(dw_ih), _parr(dw_hh),
            _parr(db_ih), _parr(db_hh), _stream(stream))
    if lengths is None:
        return lib.lstm_backward(ctypes.byref(desc), *args)
    return lib.lstm_backward_varlen(ctypes.byref(desc), _p(lengths), *args)


def lstm_forward_noalloc(desc, x, h0, c0, w_ih, w_hh, b_ih, b_hh, out, h_n, c_n,
                         stream=None) -> int:
    lib = load()
    return lib.lstm_forward_noalloc(ctypes.byref(desc), _p(x), _p(h0), _p(c0), _parr(w_ih),
                                    _parr(w_hh), _parr(b_ih), _parr(b_hh), _p(out), _p(h_n),
                                    _p(c_n), _stream(stream))


def lstm_noalloc_query_status(stream=None) -> int:
    return int(load().lstm_noalloc_query_status(_stream(stream)))


def lstm_query_status(workspace, stream=None) -> int:
    return int(load().lstm_query_status(_p(workspace), _stream(stream)))


def lstm_timing_enable(enable: bool) -> int:
    return int(load().lstm_timing_enable(int(bool(enable))))


def lstm_timing_reset() -> None:
    load().lstm_timing_reset()


def lstm_timing_read() -> dict:
    """{kind: (launches, total_ms)} accumulated since the last reset."""
    lib = load()
    n = lib.lstm_timing_read(None, 0)
    arr = (lstm_kernel_time * n)()
    got = lib.lstm_timing_read(arr, n)
    if got < 0:
        raise LstmError(LSTM_ERR_CUDA, "lstm_timing_read")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(got)}


def lstm_trace_enable(enable: bool) -> int:
    return int(load().lstm_trace_enable(int(bool(enable))))


def lstm_trace_read(max_steps: int = LSTM_TRACE_MAX_STEPS):
    """(kind, rows): rows is a list of LSTM_TRACE_EVENTS-long lists of
    %globaltimer stamps (ns) of the last traced recurrent launch."""
    lib = load()
    buf = (ctypes.c_ulonglong * (max_steps * LSTM_TRACE_EVENTS))()
    kind = ctypes.c_int(0)
    n = lib.lstm_trace_read(buf, max_steps, ctypes.byref(kind))
    if n < 0:
        raise LstmError(LSTM_ERR_CUDA, "lstm_trace_read")
    rows = [list(buf[i * LSTM_TRACE_EVENTS:(i + 1) * LSTM_TRACE_EVENTS]) for i in range(n)]
    return int(kind.value), rows


def check(status: int, where: str = "lstm") -> None:
    if status != LSTM_OK:
        raise LstmError(status, where)
