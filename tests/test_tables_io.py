"""Routing tables and placements saved between refits and reloaded bit for
bit (CPU only)."""
import numpy as np
import pytest
import torch

import oracle
from combine_warp_top_router_b200 import synth, tables


def test_round_trip(tmp_path):
    T, E, k, R = 512, 32, 4, 8
    a = oracle.route_topk(synth.normal_f32(T, E, 1, 1).numpy(), k)[0]
    b = oracle.route_topk(synth.normal_f32(T, E, 2, 1).numpy(), k)[0]
    W, C = oracle.coselect(a, b, E)
    p = oracle.place_correlated(W, R)
    path = str(tmp_path / "tables.npz")
    # int32 views (as the device binding returns them) are stored as uint32
    tables.save_tables(path, W=torch.from_numpy(W.view(np.int32)), C=C, expert_to_rank=p,
                       meta={"step": 1000, "fit_tokens": T})
    got, meta = tables.load_tables(path)
    assert meta == {"step": 1000, "fit_tokens": T}
    assert got["W"].dtype == np.uint32 and np.array_equal(got["W"], W)
    assert np.array_equal(got["C"], C) and np.array_equal(got["expert_to_rank"], p)
    dev, _ = tables.load_tables(path, device="cpu")
    assert dev["W"].dtype == torch.int32 and np.array_equal(dev["W"].numpy().view(np.uint32), W)


def test_rejects_unknown_tables_and_wrong_widths(tmp_path):
    with pytest.raises(ValueError):
        tables.save_tables(str(tmp_path / "x.npz"), Q=np.zeros(3, np.uint32))
    with pytest.raises(ValueError):
        tables.save_tables(str(tmp_path / "x.npz"), W=np.zeros((2, 2), np.uint64))
