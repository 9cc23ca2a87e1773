"""The layer wavefront ("LSTM Forward Computation", Stack Multiple RNN
Cells): a unidirectional stack runs layer k on chunk c of the sequence while
layer k+1 runs chunk c-1, each layer on its own stream, carrying the state
between chunks through h_n / c_n.  Against the oracle with several chunk
lengths: ragged last chunks, a one-step tail merged into the chunk before,
three layers, the training forward (its saved gates feed the backward) in
float32 and bf16, and the 2-layer workload at full size on sampled rows.
Each case runs in a fresh process with LSTM_B200_WAVEFRONT=1."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))

# (chunk, L, I, H, T, B, dtype, train, seed, sampled rows)
CASES = [
    (3, 2, 24, 40, 11, 7, "f32", 1, 701, 0),     # chunks 3,3,3,2
    (3, 3, 16, 64, 10, 16, "f32", 0, 702, 0),    # chunks 3,3,4 (one-step tail merged)
    (4, 2, 32, 128, 9, 8, "bf16", 1, 703, 0),    # bf16 training
    (2, 2, 8, 12, 5, 3, "f32", 1, 704, 0),       # chunks 2,3
    (16, 2, 256, 512, 128, 64, "f32", 0, 705, 4),  # the 2-layer workload's shape
    (16, 2, 256, 512, 128, 64, "f32", 1, 706, 3),  # and its training step
]


@pytest.mark.parametrize("case", CASES, ids=[f"C{c[0]}_L{c[1]}_H{c[3]}_T{c[4]}_{c[6]}_{'train' if c[7] else 'fwd'}"
                                             for c in CASES])
def test_wavefront_parity(case, cuda_lib):
    chunk, *args = case
    env = dict(os.environ, LSTM_B200_WAVEFRONT="1", LSTM_B200_WAVEFRONT_CHUNK=str(chunk))
    r = subprocess.run([sys.executable, os.path.join(HERE, "wavefront_check.py")] + [str(a) for a in args],
                       capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
