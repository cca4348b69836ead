"""Send matrices in the DODOCO dataset's CSV layout.

"DODOCO: MoE AlltoAll Traffic Matrices on Real Text", send_matrices.csv: one
row per (dispatch, source rank) with the columns call, step, pass, layer,
src_rank, to_rank_0 .. to_rank_{R-1}; the R rows sharing a call form one R x R
matrix, and the combine returns the same volumes transposed.  This module
only writes and reads that layout; the matrices come from md_dispatch_layout's
send_counts.
"""
from __future__ import annotations

import csv
from dataclasses import dataclass

import numpy as np


@dataclass
class SendMatrix:
    call: int
    step: int
    pass_: str        # "forward" or "recompute"
    layer: int
    counts: np.ndarray  # int64 [R, R]: counts[s, d] sent from rank s to rank d


def header(R: int) -> list[str]:
    return ["call", "step", "pass", "layer", "src_rank"] + [f"to_rank_{d}" for d in range(R)]


def write_send_matrices(path: str, matrices: list[SendMatrix]) -> None:
    """Write the matrices, one row per source rank, in call order."""
    if not matrices:
        raise ValueError("no send matrices")
    R = matrices[0].counts.shape[0]
    with open(path, "w", newline="") as f:
        out = csv.writer(f)
        out.writerow(header(R))
        for m in matrices:
            c = np.asarray(m.counts)
            if c.shape != (R, R):
                raise ValueError(f"call {m.call}: matrix is {c.shape}, expected {(R, R)}")
            for s in range(R):
                out.writerow([m.call, m.step, m.pass_, m.layer, s] + [int(v) for v in c[s]])


def read_send_matrices(path: str) -> list[SendMatrix]:
    """Read a send_matrices.csv back into one SendMatrix per call."""
    with open(path, newline="") as f:
        rows = list(csv.reader(f))
    head, body = rows[0], rows[1:]
    R = len(head) - 5
    if head != header(R):
        raise ValueError("not a send_matrices.csv header")
    out: dict[int, SendMatrix] = {}
    for r in body:
        call, step, pass_, layer, src = int(r[0]), int(r[1]), r[2], int(r[3]), int(r[4])
        m = out.setdefault(call, SendMatrix(call, step, pass_, layer, np.zeros((R, R), np.int64)))
        m.counts[src] = [int(v) for v in r[5:]]
    return [out[c] for c in sorted(out)]
