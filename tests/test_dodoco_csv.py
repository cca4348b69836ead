"""The DODOCO send_matrices.csv layout ("DODOCO: MoE AlltoAll Traffic Matrices
on Real Text", send_matrices.csv columns): written and read back on the CPU.
The matrices here come from the oracle's layout, so the file also carries its
invariants (conventional rows sum to T_r * k)."""
import csv

import numpy as np
import pytest

import oracle
from combine_warp_top_router_b200 import dodoco, synth


def _matrices():
    out = []
    for call, (mode, layer) in enumerate([(0, 0), (1, 0), (0, 1)]):
        T, E, k, R = 16 * 64, 64, 6, 16
        lg = synth.normal_f32(T, E, call, 1).numpy()
        idx = oracle.route_topk(lg, k)[0]
        L = oracle.dispatch_layout(idx, E, R, synth.contiguous_placement(E, R).numpy(), mode)
        out.append(dodoco.SendMatrix(call, 6 + call, "forward", layer, L["send_counts"].reshape(R, R)))
    return out


def test_header_and_rows(tmp_path):
    path = tmp_path / "send_matrices.csv"
    ms = _matrices()
    dodoco.write_send_matrices(str(path), ms)
    rows = list(csv.reader(open(path)))
    assert rows[0][:5] == ["call", "step", "pass", "layer", "src_rank"]
    assert rows[0][5:] == [f"to_rank_{d}" for d in range(16)]
    assert len(rows) == 1 + 16 * len(ms)
    # conventional dispatch: every source rank sends T_r * k assignments
    for r in rows[1:17]:
        assert sum(int(v) for v in r[5:]) == 64 * 6


def test_round_trip(tmp_path):
    path = tmp_path / "send_matrices.csv"
    ms = _matrices()
    dodoco.write_send_matrices(str(path), ms)
    back = dodoco.read_send_matrices(str(path))
    assert [(m.call, m.step, m.pass_, m.layer) for m in back] == \
        [(m.call, m.step, m.pass_, m.layer) for m in ms]
    for a, b in zip(back, ms):
        assert np.array_equal(a.counts, b.counts)


def test_rejects_ragged_matrix(tmp_path):
    ms = _matrices()
    ms[1].counts = ms[1].counts[:3]
    with pytest.raises(ValueError):
        dodoco.write_send_matrices(str(tmp_path / "x.csv"), ms)
