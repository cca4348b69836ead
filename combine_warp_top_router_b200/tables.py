"""Save and reload the fitted routing tables and placements.

"Expert Coupling in MoE Pretraining" (PicX summary), Correlation Formation and
Stability: correlation tables fitted on a few thousand tokens stay valid, and
refitting every ~1000 steps is expected to suffice.  Between refits a run keeps
its tables and placements; this module writes them to one .npz file (counts
as uint32, placements as int32, plus a small JSON header) and reads them back
bit for bit.
"""
from __future__ import annotations

import json

import numpy as np
import torch

_KINDS = {"W": np.uint32, "C": np.uint32, "C2": np.uint32, "expert_to_rank": np.int32}


def _host(a, dtype):
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    a = np.ascontiguousarray(a)
    if a.dtype.itemsize != np.dtype(dtype).itemsize:
        raise ValueError(f"expected {np.dtype(dtype).itemsize}-byte elements, got {a.dtype}")
    return a.view(dtype)


def save_tables(path: str, meta: dict | None = None, **tables) -> None:
    """save_tables(path, W=..., C=..., C2=..., expert_to_rank=..., meta={...}).

    Device tensors are copied to the host; int32 views of uint32 counts (as the
    binding returns them) are stored as uint32."""
    unknown = set(tables) - set(_KINDS)
    if unknown:
        raise ValueError(f"unknown tables {sorted(unknown)}")
    arrays = {k: _host(v, _KINDS[k]) for k, v in tables.items() if v is not None}
    header = json.dumps({"format": 1, "tables": sorted(arrays), "meta": meta or {}})
    np.savez(path, __header__=np.frombuffer(header.encode(), np.uint8), **arrays)


def load_tables(path: str, device=None) -> tuple[dict, dict]:
    """-> (tables, meta); tables as numpy arrays, or int32 tensors on `device`."""
    with np.load(path) as z:
        header = json.loads(bytes(z["__header__"]).decode())
        out = {k: z[k].copy() for k in header["tables"]}
    if device is not None:
        out = {k: torch.from_numpy(v.view(np.int32)).to(device) for k, v in out.items()}
    return out, header["meta"]
