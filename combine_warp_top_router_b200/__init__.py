"""B200-native MoE token dispatch / combine for expert parallelism.

The compute lives in libmoedispatch.so (hand-written sm_100a CUDA kernels
behind the C ABI in include/moedispatch.h).  `binding` is a thin ctypes layer
with the same entry-point names; `synth` draws seeded synthetic inputs;
`dodoco` writes send matrices in the DODOCO dataset's CSV layout; `tables`
saves and reloads fitted count tables and placements between refits.
"""
from .binding import *  # noqa: F401,F403
from .binding import (Layout, MoeDispatchError, check_status, lib, new_status,  # noqa: F401
                      pearson_from_sums, table1_row)
from . import dodoco, synth, tables  # noqa: F401

__all__ = [n for n in dir() if n.startswith("md_") or n.startswith("MD_")] + [
    "Layout", "MoeDispatchError", "check_status", "lib", "new_status", "pearson_from_sums",
    "table1_row", "dodoco", "synth", "tables"]
