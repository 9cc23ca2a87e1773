"""Builds and runs the tcgen05.mma issue-cost probe (csrc/mma_issue_probe.cu).

    python -m layer_lstm_b200.mma_probe            # needs a B200

A measurement tool beside the library, not part of it.  It prints the
probe's CSV and then, per loop shape, N and number of issuing warps, the
marginal cost of one MMA: the cycles of a 64-MMA chain minus those of a
16-MMA chain, over the 48 MMAs in between (per issuing warp).  At M = 128,
K = 16 the tensor pipe's own rate is N / 2 cycles per MMA (4096 bf16
multiply-adds per clock per SM); above it the issuing thread is the limit.
"""
import csv
import io
import os
import subprocess
import sys
import tempfile

from . import build as _build

SRC = os.path.join(_build.CSRC, "mma_issue_probe.cu")

SHAPES = {0: "A in shared memory (ss)", 1: "A in tensor memory (ts)", 2: "ss and ts in one loop, ss taken",
          3: "ss and ts in one loop, ts taken", 4: "ts loop then ss loop",
          5: "ts, wait + fence + commit per 4 MMAs", 6: "ts, commit per 4 MMAs", 7: "ts, wait + fence per 4 MMAs",
          8: "ts, wait per 4 MMAs", 9: "ts, fence per 4 MMAs", 10: "ts, relaxed wait + fence per 4 MMAs",
          11: "ts, test_wait + fence per 4 MMAs", 12: "waits alone (no MMA)", 13: "ts, shared load per 4 MMAs",
          14: "waits alone, iteration-bounded", 15: "globaltimer reads alone",
          16: "arrive then wait on the fresh phase, alone", 17: "waits alone, whole warp",
          18: "waits alone, try_wait with a suspend-time hint",
          19: "ts, wait per 4 MMAs by the whole warp, lane 0 issues",
          20: "ts, wait per 4 MMAs by the whole warp, elect.sync issues"}


def marginal(rows):
    """{(mode, N, warps): cycles per MMA} from the 16- and 64-MMA chains
    (median of the repetitions)."""
    cyc = {}
    for r in rows:
        reps = sorted(int(r[k]) for k in ("cyc_rep1", "cyc_rep2", "cyc_rep3"))
        cyc[(int(r["mode"]), int(r["N"]), int(r["warps"]), int(r["nmma_per_warp"]))] = reps[1]
    out = {}
    for (mode, n, w, k), c in cyc.items():
        if k == 64 and (mode, n, w, 16) in cyc:
            out[(mode, n, w)] = (c - cyc[(mode, n, w, 16)]) / 48.0
    return out


def main() -> int:
    exe = os.path.join(tempfile.mkdtemp(prefix="mma_probe_"), "mma_issue_probe")
    subprocess.run([_build.NVCC, "-O2"] + _build.ARCH + ["-o", exe, SRC], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    sys.stdout.write(r.stdout)
    if r.returncode != 0:
        sys.stderr.write(r.stderr)
        return r.returncode
    rows = list(csv.DictReader(io.StringIO("\n".join(l for l in r.stdout.splitlines() if "," in l))))
    print("\nshape | N | issuing warps | cycles per MMA (per warp) | tensor-pipe rate")
    for (mode, n, w), c in sorted(marginal(rows).items()):
        print(f"{SHAPES[mode]} | {n} | {w} | {c:.1f} | {n / 2:.0f}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
