"""The oracle: a plain, slow CPU statement of the MoE dispatch / combine path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never calls it and shares no code with it.

The arithmetic lives in ``moe_oracle.c`` (plain C, single-threaded).  This
module compiles it on first use with gcc and marshals numpy arrays to it; it
holds no arithmetic of its own.  Every function takes and returns numpy arrays.

Sources (page title -- section), cited per function in ``moe_oracle.c``:
  "Expert Coupling in MoE Pretraining ..." (PicX summary): Background; Method 1
    (deduplicating dispatcher, correlated placement); Method 2 (token shuffling).
  "DODOCO: MoE AlltoAll Traffic Matrices on Real Text": Setup; send_matrices.csv;
    Reading the counts.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CONV, DEDUP = 0, 1
GATE_TOPK_SOFTMAX, GATE_FULL_SOFTMAX = 0, 1
COMBINE_FUSED, COMBINE_WIRE = 0, 1


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so next to it (gcc, -O2, no fast-math)."""
    stale = not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64, I32 = ctypes.c_int64, ctypes.c_int
            lib.oracle_route_topk.argtypes = [P, I64, I32, I32, I32, P, P]
            lib.oracle_dispatch_layout.argtypes = [P, I64, I32, I32, I32, P, I32,
                                                   P, P, P, P, P, P, P, P, P]
            lib.oracle_dispatch_permute.argtypes = [P, I64, I64, P, I64, P]
            lib.oracle_dedup_expand.argtypes = [P, I64, I64, P, P, I64, I32, I64, P]
            lib.oracle_combine.argtypes = [P, I64, P, P, P, I64, I32, I64, I32, P, I32, P, P, P]
            lib.oracle_coselect.argtypes = [P, P, I64, I32, I32, P, P, I32]
            lib.oracle_placement_objective.argtypes = [P, I32, P]
            lib.oracle_placement_objective.restype = ctypes.c_longlong
            lib.oracle_place_correlated.argtypes = [P, I32, I32, I32, I32, P]
            lib.oracle_token_shuffle.argtypes = [P, P, P, I64, I32, I32, I32, P, P, P]
            lib.oracle_coselect_pair.argtypes = [P, P, P, I64, I32, I32, P]
            lib.oracle_rank_stats.argtypes = [P, I64, I32, I32, I32, P, P]
            lib.oracle_successor_share.argtypes = [P, P, I32, P, P]
            lib.oracle_count_sums.argtypes = [P, P, I64, P]
            lib.oracle_place_two_level.argtypes = [P, I32, I32, I32, I32, I32, P]
            lib.oracle_token_shuffle_rounds.argtypes = [P, P, P, I64, I32, I32, I32, P, P, P, P]
            lib.oracle_token_shuffle_pair.argtypes = [P, P, P, P, P, I64, I32, I32, I32,
                                                      ctypes.c_uint64, P, P, P, P]
            for name in ("oracle_route_topk", "oracle_dispatch_layout", "oracle_dispatch_permute",
                         "oracle_dedup_expand",
                         "oracle_combine", "oracle_coselect", "oracle_place_correlated",
                         "oracle_token_shuffle", "oracle_coselect_pair",
                         "oracle_token_shuffle_pair", "oracle_rank_stats",
                         "oracle_successor_share", "oracle_count_sums",
                         "oracle_place_two_level", "oracle_token_shuffle_rounds"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def route_topk(logits, k, gate_mode=GATE_TOPK_SOFTMAX):
    """logits float32 [T, E] -> (idx int32 [T, k], w float32 [T, k])."""
    lib = _load()
    lg = _c(logits, np.float32)
    T, E = lg.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _check(lib.oracle_route_topk(_ptr(lg), T, E, k, gate_mode, _ptr(idx), _ptr(w)), "route_topk")
    return idx, w


def dispatch_layout(idx, E, R, expert_to_rank, mode):
    """Returns a dict with the layout outputs (see moe_oracle.c)."""
    lib = _load()
    ix = _c(idx, np.int32)
    T, k = ix.shape
    p = _c(expert_to_rank, np.int32)
    cap = T * k
    out = dict(
        row_of_slot=np.full((T, k), -1, np.int32),
        assign_row=np.full((T, k), -1, np.int32),
        row_token=np.full(max(cap, 1), -1, np.int32),
        row_mask=np.zeros(max(cap, 1), np.uint32),
        send_counts=np.zeros((R, R), np.int64),
        expert_counts=np.zeros(E, np.int64),
        expert_offsets=np.zeros(E + 1, np.int64),
        rank_offsets=np.zeros(R + 1, np.int64),
    )
    n = np.zeros(1, np.int64)
    rc = lib.oracle_dispatch_layout(
        _ptr(ix), T, E, k, R, _ptr(p), mode, _ptr(out["row_of_slot"]), _ptr(out["assign_row"]),
        _ptr(out["row_token"]), _ptr(out["row_mask"]), _ptr(out["send_counts"]),
        _ptr(out["expert_counts"]), _ptr(out["expert_offsets"]), _ptr(out["rank_offsets"]), _ptr(n))
    _check(rc, "dispatch_layout")
    n_rows = int(n[0])
    out["n_rows"] = n_rows
    out["row_token"] = out["row_token"][:n_rows]
    out["row_mask"] = out["row_mask"][:n_rows]
    return out


def dispatch_permute(x_bits, row_token):
    """x_bits uint16 [T, H] (bf16 bit patterns) -> out uint16 [n_rows, H]."""
    lib = _load()
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    rt = _c(row_token, np.int32)
    out = np.empty((rt.shape[0], H), np.uint16)
    _check(lib.oracle_dispatch_permute(_ptr(x), T, H, _ptr(rt), rt.shape[0], _ptr(out)), "permute")
    return out


def dedup_expand(wire_bits, row_of_slot, assign_row, n_out=None):
    """Receiver-side expand: out[assign_row[t, j]] = wire[row_of_slot[t, j]].

    wire_bits uint16 [n_wire, H]; row_of_slot, assign_row int32 [T, k] ->
    out uint16 [n_out, H] (n_out defaults to T * k)."""
    lib = _load()
    wire = _c(wire_bits, np.uint16)
    n_wire, H = wire.shape
    rs = _c(row_of_slot, np.int32)
    ar = _c(assign_row, np.int32)
    T, k = rs.shape
    n_out = T * k if n_out is None else int(n_out)
    out = np.zeros((n_out, H), np.uint16)
    _check(lib.oracle_dedup_expand(_ptr(wire), n_wire, H, _ptr(rs), _ptr(ar), T, k, n_out, _ptr(out)),
           "dedup_expand")
    return out


def combine(y_bits, assign_row, idx, w, mode=COMBINE_FUSED, expert_to_rank=None,
            row_of_slot=None, z_rows=0):
    """y_bits uint16 [rows, H] -> out uint16 [T, H] (and z uint16 [z_rows, H] for WIRE)."""
    lib = _load()
    y = _c(y_bits, np.uint16)
    ar = _c(assign_row, np.int32)
    ix = _c(idx, np.int32)
    ww = _c(w, np.float32)
    T, k = ix.shape
    H = y.shape[1]
    out = np.empty((T, H), np.uint16)
    z = None
    p = R = rs = None
    if mode == COMBINE_WIRE:
        p = _c(expert_to_rank, np.int32)
        rs = _c(row_of_slot, np.int32)
        z = np.zeros((max(z_rows, 1), H), np.uint16)
    rc = lib.oracle_combine(_ptr(y), y.shape[0], _ptr(ar), _ptr(ix), _ptr(ww), T, k, H, mode,
                            _ptr(p), 0 if p is None else int(p.max(initial=0)) + 1, _ptr(rs),
                            _ptr(z), _ptr(out))
    _check(rc, "combine")
    if mode == COMBINE_WIRE:
        return out, z[:z_rows]
    return out


def coselect(idx_l, idx_next, E, T_fit=None, want_W=True, want_C=True):
    """Returns (W, C) uint32 [E, E] counted over tokens [0, T_fit)."""
    lib = _load()
    a = _c(idx_l, np.int32)
    T, k = a.shape
    T_fit = T if T_fit is None else T_fit
    b = None if idx_next is None else _c(idx_next, np.int32)
    W = np.zeros((E, E), np.uint32) if want_W else None
    C = np.zeros((E, E), np.uint32) if (want_C and b is not None) else None
    _check(lib.oracle_coselect(_ptr(a), _ptr(b), T_fit, E, k, _ptr(W), _ptr(C), 0), "coselect")
    return W, C


def placement_objective(W, expert_to_rank):
    lib = _load()
    Wc = _c(W, np.uint32)
    p = _c(expert_to_rank, np.int32)
    return int(lib.oracle_placement_objective(_ptr(Wc), Wc.shape[0], _ptr(p)))


def place_correlated(W, R, seed_mode=0, refine=True):
    """W uint32 [E, E] (symmetric) -> expert_to_rank int32 [E]."""
    lib = _load()
    Wc = _c(W, np.uint32)
    E = Wc.shape[0]
    p = np.empty(E, np.int32)
    _check(lib.oracle_place_correlated(_ptr(Wc), E, R, seed_mode, 1 if refine else 0, _ptr(p)),
           "place_correlated")
    return p


def token_shuffle(idx_l, C, expert_to_rank_next, R):
    """Returns (pred_rank, perm, inv), each int32 [T]."""
    lib = _load()
    a = _c(idx_l, np.int32)
    T, k = a.shape
    Cc = _c(C, np.uint32)
    E = Cc.shape[0]
    p = _c(expert_to_rank_next, np.int32)
    pred = np.empty(T, np.int32)
    perm = np.empty(T, np.int32)
    inv = np.empty(T, np.int32)
    _check(lib.oracle_token_shuffle(_ptr(a), _ptr(Cc), _ptr(p), T, E, k, R,
                                    _ptr(pred), _ptr(perm), _ptr(inv)), "token_shuffle")
    return pred, perm, inv


def coselect_pair(idx_prev, idx_l, idx_next, E, T_fit=None):
    """Pair counts C2[a, b, e'] over the first T_fit tokens: uint32 [E, E, E]."""
    lib = _load()
    a = _c(idx_prev, np.int32)
    b = _c(idx_l, np.int32)
    c = _c(idx_next, np.int32)
    T, k = b.shape
    T_fit = T if T_fit is None else int(T_fit)
    C2 = np.empty((E, E, E), np.uint32)
    _check(lib.oracle_coselect_pair(_ptr(a), _ptr(b), _ptr(c), T_fit, E, k, _ptr(C2)), "coselect_pair")
    return C2


def token_shuffle_pair(idx_prev, idx_l, C, C2, expert_to_rank_next, R, min_obs):
    """Pair-based prediction with single-expert fallback -> (pred, perm, inv, use_pair)."""
    lib = _load()
    a = _c(idx_prev, np.int32)
    b = _c(idx_l, np.int32)
    T, k = b.shape
    E = C.shape[0]
    Cc = _c(C, np.uint32)
    C2c = _c(C2, np.uint32)
    pn = _c(expert_to_rank_next, np.int32)
    pred = np.empty(T, np.int32)
    perm = np.empty(T, np.int32)
    inv = np.empty(T, np.int32)
    use = np.empty(T, np.int32)
    _check(lib.oracle_token_shuffle_pair(_ptr(a), _ptr(b), _ptr(Cc), _ptr(C2c), _ptr(pn), T, E, k, R,
                                         int(min_obs), _ptr(pred), _ptr(perm), _ptr(inv), _ptr(use)),
           "token_shuffle_pair")
    return pred, perm, inv, use


def rank_stats(idx, E, R, expert_to_rank):
    """hist int64 [k+1]: tokens with exactly D distinct destination ranks."""
    lib = _load()
    ix = _c(idx, np.int32)
    T, k = ix.shape
    p = _c(expert_to_rank, np.int32)
    hist = np.zeros(k + 1, np.int64)
    _check(lib.oracle_rank_stats(_ptr(ix), T, E, k, R, _ptr(p), _ptr(hist)), "rank_stats")
    return hist


def successor_share(C, W):
    """(num uint32 [E], den uint32 [E]): largest C[e, :] and W[e, e]."""
    lib = _load()
    Cc = _c(C, np.uint32)
    Wc = _c(W, np.uint32)
    E = Cc.shape[0]
    num = np.empty(E, np.uint32)
    den = np.empty(E, np.uint32)
    _check(lib.oracle_successor_share(_ptr(Cc), _ptr(Wc), E, _ptr(num), _ptr(den)), "successor_share")
    return num, den


def count_sums(x, y):
    """Exact (sx, sy, sxx, syy, sxy) of two uint32 count tables, as Python ints."""
    lib = _load()
    xc = _c(np.ravel(x), np.uint32)
    yc = _c(np.ravel(y), np.uint32)
    out = np.zeros(10, np.uint64)
    _check(lib.oracle_count_sums(_ptr(xc), _ptr(yc), xc.shape[0], _ptr(out)), "count_sums")
    return tuple(int(out[2 * i]) | (int(out[2 * i + 1]) << 64) for i in range(5))


def pearson(x, y):
    """Pearson correlation of two count tables from their exact sums."""
    n = int(np.size(x))
    sx, sy, sxx, syy, sxy = count_sums(x, y)
    cov = n * sxy - sx * sy
    vx = n * sxx - sx * sx
    vy = n * syy - sy * sy
    return cov / (vx * vy) ** 0.5 if vx > 0 and vy > 0 else float("nan")


REFINE_NONE, REFINE_SWAPS, REFINE_KL = 0, 1, 2


def place_two_level(W, R, nodes=1, seed_mode=0, refine_mode=REFINE_SWAPS):
    """Placement over `nodes` nodes of R/nodes ranks (nodes=1: one level), with
    no refinement, best single swaps, or Kernighan-Lin passes."""
    lib = _load()
    Wc = _c(W, np.uint32)
    E = Wc.shape[0]
    p = np.empty(E, np.int32)
    _check(lib.oracle_place_two_level(_ptr(Wc), E, R, nodes, seed_mode, refine_mode, _ptr(p)),
           "place_two_level")
    return p


def token_shuffle_rounds(idx_l, C, expert_to_rank_next, R):
    """Rounds-based capacity assignment -> (pred, perm, inv, rounds)."""
    lib = _load()
    ix = _c(idx_l, np.int32)
    T, k = ix.shape
    Cc = _c(C, np.uint32)
    E = Cc.shape[0]
    pn = _c(expert_to_rank_next, np.int32)
    pred = np.empty(T, np.int32)
    perm = np.empty(T, np.int32)
    inv = np.empty(T, np.int32)
    rounds = np.zeros(1, np.int32)
    _check(lib.oracle_token_shuffle_rounds(_ptr(ix), _ptr(Cc), _ptr(pn), T, E, k, R, _ptr(pred),
                                           _ptr(perm), _ptr(inv), _ptr(rounds)), "token_shuffle_rounds")
    return pred, perm, inv, int(rounds[0])
