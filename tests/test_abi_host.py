"""Host-side checks of the C-ABI library: it builds, loads, exports every
function include/lstm.h declares, sizes its buffers, and rejects bad
arguments before touching a GPU (the warp_nn page's ValueError cases map to
LSTM_ERR_INVALID_ARG).  No compute call runs here."""
import ctypes
import os
import re
import subprocess

import pytest

from layer_lstm_b200 import binding
from layer_lstm_b200.build import LIB_PATH

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(lstm_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    binding.load()
    declared = _declared_functions()
    assert set(binding.EXPORTED) <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\b(lstm_[a-z_0-9]+)\b", out))
    missing = [n for n in declared if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(LIB_PATH)
    for n in declared:
        getattr(lib, n)


def test_status_strings():
    for code, name in [(0, "LSTM_OK"), (1, "LSTM_ERR_INVALID_ARG"), (2, "LSTM_ERR_UNSUPPORTED"),
                       (3, "LSTM_ERR_WORKSPACE"), (4, "LSTM_ERR_CUDA"), (5, "LSTM_ERR_TIMEOUT")]:
        assert binding.lstm_status_string(code) == name


def test_size_queries():
    d = binding.make_desc(256, 512, 2, False, True, True, 64, 128, binding.LSTM_F32)
    ws = binding.lstm_workspace_size(d)
    rs = binding.lstm_reserve_size(d)
    T, B, H, G = 128, 64, 512, 2048
    # reserve: per layer gates (T*B*G) + c (T*B*H) float32 + the output sequence
    assert rs >= 2 * (T * B * G * 4 + T * B * H * 4 + T * B * H * 4)
    assert ws >= T * B * G * 4   # at least the projection output
    # bf16 halves the stored sequences
    d16 = binding.make_desc(256, 512, 2, False, True, True, 64, 128, binding.LSTM_BF16)
    assert binding.lstm_reserve_size(d16) < rs


@pytest.mark.parametrize("field,value", [("num_layers", 0), ("hidden_size", 0), ("input_size", 0),
                                         ("batch", -1), ("seq_len", -1), ("dtype", 7),
                                         ("bidirectional", 2)])
def test_invalid_desc(field, value):
    d = binding.make_desc(8, 16, 1, False, True, True, 4, 5)
    setattr(d, field, value)
    assert binding.lstm_workspace_size(d) == 0
    assert binding.lstm_reserve_size(d) == 0
    dummy = [1]
    st = binding.lstm_forward(d, 1, None, None, dummy, dummy, dummy, dummy, 1, 1, 1, 256,
                              stream=0, ws_bytes=1 << 30)
    assert st == binding.LSTM_ERR_INVALID_ARG


def test_null_pointers_rejected():
    d = binding.make_desc(8, 16, 1, False, True, True, 4, 5)
    one = [256]
    # missing weights
    assert binding.lstm_forward(d, 256, None, None, None, one, one, one, 256, 256, 256, 256,
                                stream=0, ws_bytes=1 << 30) == binding.LSTM_ERR_INVALID_ARG
    # missing bias with bias=1
    assert binding.lstm_forward(d, 256, None, None, one, one, None, None, 256, 256, 256, 256,
                                stream=0, ws_bytes=1 << 30) == binding.LSTM_ERR_INVALID_ARG
    # missing x
    assert binding.lstm_forward(d, None, None, None, one, one, one, one, 256, 256, 256, 256,
                                stream=0, ws_bytes=1 << 30) == binding.LSTM_ERR_INVALID_ARG
    # misaligned workspace
    assert binding.lstm_forward(d, 256, None, None, one, one, one, one, 256, 256, 256, 257,
                                stream=0, ws_bytes=1 << 30) == binding.LSTM_ERR_INVALID_ARG
    # backward without reserve
    assert binding.lstm_backward(d, 256, None, None, one, one, 256, None, None, None, 256,
                                 256, 256, 256, one, one, one, one, stream=0,
                                 ws_bytes=1 << 30, rs_bytes=0) == binding.LSTM_ERR_INVALID_ARG


def test_workspace_too_small():
    d = binding.make_desc(8, 16, 1, False, True, True, 4, 5)
    one = [256]
    need = binding.lstm_workspace_size(d)
    st = binding.lstm_forward(d, 256, None, None, one, one, one, one, 256, 256, 256, 256,
                              stream=0, ws_bytes=need - 1)
    assert st == binding.LSTM_ERR_WORKSPACE


def test_bf16_backward_checks_workspace():
    """bf16 backward is implemented (float32 staging in the workspace): an
    undersized workspace is refused before anything is enqueued."""
    d = binding.make_desc(8, 16, 1, False, True, True, 4, 5, binding.LSTM_BF16)
    one = [256]
    need = binding.lstm_workspace_size(d)
    st = binding.lstm_backward(d, 256, None, None, one, one, 256, None, None, 256, 256,
                               256, 256, 256, one, one, one, one, stream=0,
                               ws_bytes=need - 1, rs_bytes=1 << 30)
    assert st == binding.LSTM_ERR_WORKSPACE
