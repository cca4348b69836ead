"""Thin ctypes binding of libmoedispatch (include/moedispatch.h).

Argument marshalling only: every function checks tensor placement, dtype and
contiguity, allocates outputs with torch when the caller passes none, and calls
the C entry point of the same name on the current CUDA stream.  All arithmetic
runs in the library's kernels.  If libmoedispatch.so is missing the first call
raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoedispatch.so")

MD_OK, MD_ERR_ARG, MD_ERR_UNSUPPORTED, MD_ERR_CUDA = 0, 1, 2, 3
MD_ERR_WORKSPACE, MD_ERR_DATA, MD_ERR_TIMEOUT = 4, 5, 6
MD_CONV, MD_DEDUP = 0, 1
MD_GATE_TOPK_SOFTMAX, MD_GATE_FULL_SOFTMAX = 0, 1
MD_COMBINE_FUSED, MD_COMBINE_WIRE = 0, 1
MD_SEED_CONTIGUOUS, MD_SEED_GREEDY_PAIRS = 0, 1
MD_REFINE_NONE, MD_REFINE_SWAPS, MD_REFINE_KL = 0, 1, 2
MD_PERMUTE_AUTO, MD_PERMUTE_BULK, MD_PERMUTE_VECTOR = 0, 1, 2
MD_LAYOUT_AUTO, MD_LAYOUT_COOPERATIVE, MD_LAYOUT_SPLIT = 0, 1, 2

_lock = threading.Lock()
_lib = None

_P, _I, _L, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_SIGNATURES = {
    "md_status_string": ([_I], ctypes.c_char_p),
    "md_version": ([], _I),
    "md_launch_count": ([], ctypes.c_uint64),
    "md_memset_count": ([], ctypes.c_uint64),
    "md_route_topk": ([_P, _L, _I, _I, _I, _P, _P, _P], _I),
    "md_dispatch_layout_workspace_size": ([_L, _I, _I, _I, _I], _S),
    "md_dispatch_layout": ([_P, _L, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                            _P, _S, _P, _P], _I),
    "md_dispatch_layout_noalloc_max_scratch": ([], _S),
    "md_dispatch_layout_noalloc": ([_P, _L, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                                    _P, _P, _P], _I),
    "md_dispatch_permute": ([_P, _L, _I, _I, _P, _L, _P, _P, _P], _I),
    "md_set_permute_path": ([_I], _I),
    "md_set_layout_path": ([_I], _I),
    "md_exchange_plan": ([_P, _I, _I, _P, _P], _I),
    "md_dispatch_exchange": ([_P, _L, _I, _I, _P, _P, _P, _I, _I, _P, _P, _L, _P, _P, _P], _I),
    "md_combine_partials": ([_P, _L, _P, _P, _P, _L, _I, _I, _P, _P, _P], _I),
    "md_combine_exchange": ([_P, _L, _I, _I, _P, _P, _I, _I, _P, _P, _P, _P, _P], _I),
    "md_dedup_expand": ([_P, _L, _I, _P, _P, _L, _I, _L, _P, _P, _P], _I),
    "md_combine": ([_P, _L, _P, _P, _P, _L, _I, _I, _I, _P, _L, _P, _P, _P, _P], _I),
    "md_coselect_stats": ([_P, _P, _L, _I, _I, _P, _P, _I, _P, _P], _I),
    "md_place_correlated_workspace_size": ([_I, _I], _S),
    "md_place_correlated": ([_P, _I, _I, _I, _I, _P, _P, _S, _P, _P], _I),
    "md_token_shuffle_workspace_size": ([_L, _I, _I], _S),
    "md_token_shuffle": ([_P, _I, _P, _P, _L, _I, _I, _P, _P, _P, _P, _S, _P, _P], _I),
    "md_coselect_pair_stats": ([_P, _P, _P, _L, _I, _I, _P, _I, _P, _P], _I),
    "md_token_shuffle_rounds_workspace_size": ([_L, _I, _I], _S),
    "md_token_shuffle_rounds": ([_P, _I, _P, _P, _L, _I, _I, _P, _P, _P, _P, _P, _S, _P, _P], _I),
    "md_rank_stats": ([_P, _L, _I, _I, _I, _P, _P, _P, _P], _I),
    "md_set_test_hooks": ([ctypes.c_longlong, _I, ctypes.c_longlong], None),
    "md_place_two_level_workspace_size": ([_I, _I, _I], _S),
    "md_place_two_level": ([_P, _I, _I, _I, _I, _I, _P, _P, _S, _P, _P], _I),
    "md_successor_share": ([_P, _P, _I, _P, _P, _P], _I),
    "md_count_sums": ([_P, _P, _L, _P, _P], _I),
    "md_table1_row": ([_P, _I, _P], _I),
    "md_pearson_from_sums": ([_P, _L, _P], _I),
    "md_token_shuffle_pair_workspace_size": ([_L, _I, _I], _S),
    "md_token_shuffle_pair": ([_P, _P, _I, _P, _P, _P, _L, _I, _I, ctypes.c_uint32, _P, _P, _P, _P,
                               _P, _S, _P, _P], _I),
    "md_gather_rows": ([_P, _L, _L, _P, _L, _P, _P, _P], _I),
}


class MoeDispatchError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)}")
        self.code = code


def lib():
    """The loaded libmoedispatch.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m combine_warp_top_router_b200.build` (there is no CPU fallback)")
            h = ctypes.CDLL(LIB_PATH)
            for name, (args, res) in _SIGNATURES.items():
                fn = getattr(h, name)
                fn.argtypes = args
                fn.restype = res
            _lib = h
    return _lib


def status_string(code: int) -> str:
    return lib().md_status_string(int(code)).decode()


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(lib().md_launch_count())


def memset_count() -> int:
    """Device memsets and device-to-device copies the library has enqueued."""
    return int(lib().md_memset_count())


def _check(rc: int, what: str):
    if rc != MD_OK:
        raise MoeDispatchError(rc, what)


def _call(name: str, dev, *args) -> int:
    """Call entry point `name` with `dev` as the current CUDA device.

    The CUDA runtime launches on the calling thread's current device, and the
    library looks up per-device state (kernel attributes, the allocation-free
    scratch array) for that device, so tensors on another device are handled
    by making their device current for the call."""
    fn = getattr(lib(), name)
    dev = torch.device(dev)
    if dev.index is None or torch.cuda.current_device() == dev.index:
        return fn(*args)
    with torch.cuda.device(dev):
        return fn(*args)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return t


def _room(t, name, n):
    """The kernels write by computed offsets: a buffer must hold n elements."""
    if t is not None and t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {n}")
    return t


def new_status(device) -> torch.Tensor:
    """A device status word for the dev_status arguments."""
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(dev_status: torch.Tensor, what: str = "device status"):
    """Synchronise on the status word and raise if a kernel reported an error."""
    code = int(dev_status.item())
    if code != MD_OK:
        raise MoeDispatchError(code, what)


# ------------------------------------------------------------------ router

def md_route_topk(logits, k, gate_mode=MD_GATE_TOPK_SOFTMAX, topk_idx=None, topk_w=None,
                  stream=None):
    _need(logits, "logits", torch.float32)
    T, E = logits.shape
    dev = logits.device
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _need(topk_w, "topk_w", torch.float32, dev)
    _room(topk_idx, "topk_idx", T * k)
    _room(topk_w, "topk_w", T * k)
    rc = _call("md_route_topk", dev, _ptr(logits), T, E, k, gate_mode, _ptr(topk_idx), _ptr(topk_w),
                             _stream(stream, dev))
    _check(rc, "md_route_topk")
    return topk_idx, topk_w


# ------------------------------------------------------------------ layout

@dataclass
class Layout:
    """Outputs of md_dispatch_layout (device tensors)."""
    mode: int
    row_of_slot: torch.Tensor   # int32 [T, k]
    assign_row: torch.Tensor    # int32 [T, k]
    row_token: torch.Tensor     # int32 [row capacity]
    row_mask: torch.Tensor      # int32 [row capacity] (uint32 bit patterns)
    send_counts: torch.Tensor   # int32 [R, R]
    expert_counts: torch.Tensor  # int32 [E]
    expert_offsets: torch.Tensor  # int32 [E+1]
    rank_offsets: torch.Tensor  # int32 [R+1]
    n_rows: torch.Tensor        # int32 [1]
    row_capacity: int


def _check_layout(L, T, E, k, R, mode, dev):
    """A caller's Layout must have the buffers md_dispatch_layout writes."""
    cap = T * k if mode == MD_CONV else T * min(k, R)
    for name, n in (("row_of_slot", T * k), ("assign_row", T * k), ("row_token", cap),
                    ("row_mask", cap), ("send_counts", R * R), ("expert_counts", E),
                    ("expert_offsets", E + 1), ("rank_offsets", R + 1), ("n_rows", 1)):
        t = getattr(L, name)
        _need(t, name, torch.int32, dev)
        _room(t, name, n)


def dispatch_layout_workspace_size(T, E, k, R, mode) -> int:
    return int(lib().md_dispatch_layout_workspace_size(T, E, k, R, mode))


def alloc_layout(T, E, k, R, mode, device) -> Layout:
    cap = T * k if mode == MD_CONV else T * min(k, R)
    i32 = dict(dtype=torch.int32, device=device)
    return Layout(mode=mode, row_of_slot=torch.empty(T, k, **i32),
                  assign_row=torch.empty(T, k, **i32), row_token=torch.empty(max(cap, 1), **i32),
                  row_mask=torch.empty(max(cap, 1), **i32), send_counts=torch.empty(R, R, **i32),
                  expert_counts=torch.empty(E, **i32), expert_offsets=torch.empty(E + 1, **i32),
                  rank_offsets=torch.empty(R + 1, **i32), n_rows=torch.empty(1, **i32),
                  row_capacity=cap)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def md_dispatch_layout(topk_idx, E, R, expert_to_rank, mode, out: Layout | None = None,
                       workspace=None, dev_status=None, stream=None) -> Layout:
    _need(topk_idx, "topk_idx", torch.int32)
    dev = topk_idx.device
    _need(expert_to_rank, "expert_to_rank", torch.int32, dev)
    T, k = topk_idx.shape
    if out is None:
        out = alloc_layout(T, E, k, R, mode, dev)
    _check_layout(out, T, E, k, R, mode, dev)
    need = dispatch_layout_workspace_size(T, E, k, R, mode)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    rc = _call("md_dispatch_layout", dev, 
        _ptr(topk_idx), T, E, k, R, _ptr(expert_to_rank), mode, _ptr(out.row_of_slot),
        _ptr(out.assign_row), _ptr(out.row_token), _ptr(out.row_mask), _ptr(out.send_counts),
        _ptr(out.expert_counts), _ptr(out.expert_offsets), _ptr(out.rank_offsets),
        _ptr(out.n_rows), _ptr(workspace), workspace.numel(), _ptr(dev_status),
        _stream(stream, dev))
    _check(rc, "md_dispatch_layout")
    return out


def md_dispatch_layout_noalloc(topk_idx, E, R, expert_to_rank, mode, out: Layout | None = None,
                               dev_status=None, stream=None) -> Layout:
    """md_dispatch_layout without a workspace, for callers that cannot allocate
    device memory: the library uses its own fixed 4 MiB per-GPU scratch array.
    Calls that overlap on one GPU share that array and must be serialised."""
    _need(topk_idx, "topk_idx", torch.int32)
    dev = topk_idx.device
    _need(expert_to_rank, "expert_to_rank", torch.int32, dev)
    T, k = topk_idx.shape
    if out is None:
        out = alloc_layout(T, E, k, R, mode, dev)
    _check_layout(out, T, E, k, R, mode, dev)
    rc = _call("md_dispatch_layout_noalloc", dev, 
        _ptr(topk_idx), T, E, k, R, _ptr(expert_to_rank), mode, _ptr(out.row_of_slot),
        _ptr(out.assign_row), _ptr(out.row_token), _ptr(out.row_mask), _ptr(out.send_counts),
        _ptr(out.expert_counts), _ptr(out.expert_offsets), _ptr(out.rank_offsets),
        _ptr(out.n_rows), _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_dispatch_layout_noalloc")
    return out


# --------------------------------------------------------- permute/combine

def md_dispatch_permute(x, row_of_slot, out_rows=None, out=None, dev_status=None, stream=None):
    _need(x, "x", torch.bfloat16)
    dev = x.device
    _need(row_of_slot, "row_of_slot", torch.int32, dev)
    T, H = x.shape
    k = row_of_slot.shape[1]
    if out is None:
        out = torch.empty(out_rows if out_rows is not None else T * k, H, dtype=torch.bfloat16,
                          device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if out.dim() != 2 or out.shape[1] != H:
        raise ValueError(f"out must be [rows, {H}]")
    rc = _call("md_dispatch_permute", dev, _ptr(x), T, H, k, _ptr(row_of_slot), out.shape[0], _ptr(out),
                                   _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_dispatch_permute")
    return out


def md_set_permute_path(path=MD_PERMUTE_AUTO):
    """Choose md_dispatch_permute's kernel (tests and tuning; same bits either way)."""
    _check(lib().md_set_permute_path(int(path)), "md_set_permute_path")


def md_set_layout_path(path=MD_LAYOUT_AUTO):
    """Choose md_dispatch_layout's launch form (tests; same results either way)."""
    _check(lib().md_set_layout_path(int(path)), "md_set_layout_path")


def md_dedup_expand(wire, row_of_slot, assign_row, out_rows=None, out=None, dev_status=None,
                    stream=None):
    """out[assign_row[t, j]] = wire[row_of_slot[t, j]]: dedup rows to expert-grouped rows."""
    _need(wire, "wire", torch.bfloat16)
    dev = wire.device
    _need(row_of_slot, "row_of_slot", torch.int32, dev)
    _need(assign_row, "assign_row", torch.int32, dev)
    T, k = row_of_slot.shape
    H = wire.shape[1]
    if assign_row.shape != row_of_slot.shape:
        raise ValueError("assign_row and row_of_slot differ in shape")
    if out is None:
        out = torch.empty(out_rows if out_rows is not None else T * k, H, dtype=torch.bfloat16,
                          device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if out.dim() != 2 or out.shape[1] != H:
        raise ValueError(f"out must be [rows, {H}]")
    rc = _call("md_dedup_expand", dev, _ptr(wire), wire.shape[0], H, _ptr(row_of_slot), _ptr(assign_row), T,
                               k, out.shape[0], _ptr(out), _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_dedup_expand")
    return out


def md_combine(y, assign_row, topk_idx, topk_w, mode=MD_COMBINE_FUSED, row_of_slot=None, z=None,
               out=None, dev_status=None, stream=None):
    _need(y, "y", torch.bfloat16)
    dev = y.device
    _need(assign_row, "assign_row", torch.int32, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _need(topk_w, "topk_w", torch.float32, dev)
    T, k = topk_idx.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    _room(out, "out", T * H)
    _room(assign_row, "assign_row", T * k)
    _room(topk_w, "topk_w", T * k)
    z_rows = 0
    if mode == MD_COMBINE_WIRE:
        _need(row_of_slot, "row_of_slot", torch.int32, dev)
        _need(z, "z", torch.bfloat16, dev)
        _room(row_of_slot, "row_of_slot", T * k)
        z_rows = z.shape[0]
    rc = _call("md_combine", dev, _ptr(y), y.shape[0], _ptr(assign_row), _ptr(topk_idx), _ptr(topk_w), T,
                          k, H, mode, _ptr(row_of_slot), z_rows, _ptr(z), _ptr(out),
                          _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_combine")
    return out


def md_gather_rows(src, index, out=None, dev_status=None, stream=None):
    if not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous CUDA tensor")
    dev = src.device
    _need(index, "index", torch.int32, dev)
    n = index.shape[0]
    if out is None:
        out = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=dev)
    if out.dtype != src.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor of src's dtype")
    _room(out, "out", n * (src[0].numel() if src.shape[0] else out[0].numel()))
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else \
        out[0].numel() * out.element_size()
    rc = _call("md_gather_rows", dev, _ptr(src), src.shape[0], row_bytes, _ptr(index), n, _ptr(out),
                              _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_gather_rows")
    return out


# --------------------------------------------------- statistics / planning

def md_coselect_stats(idx_l, idx_next, E, T_fit=None, W=None, C=None, accumulate=False,
                      want_W=True, want_C=True, dev_status=None, stream=None):
    _need(idx_l, "idx_l", torch.int32)
    dev = idx_l.device
    T, k = idx_l.shape
    T_fit = T if T_fit is None else T_fit
    if idx_next is not None:
        _need(idx_next, "idx_next", torch.int32, dev)
    if W is None and want_W:
        W = torch.empty(E, E, dtype=torch.int32, device=dev)
    if C is None and want_C and idx_next is not None:
        C = torch.empty(E, E, dtype=torch.int32, device=dev)
    if C is not None and idx_next is None:
        raise ValueError("C needs idx_next (the layer-l+1 top-k)")
    if idx_next is not None and idx_next.shape[1] != k:
        raise ValueError("idx_l and idx_next differ in k")
    if idx_next is not None and idx_next.shape[0] < T_fit:
        raise ValueError("idx_next has fewer than T_fit rows")
    if T_fit > T:
        raise ValueError("T_fit exceeds the rows of idx_l")
    for t, n in ((W, "W"), (C, "C")):
        if t is not None:
            _need(t, n, torch.int32, dev)
            _room(t, n, E * E)
    rc = _call("md_coselect_stats", dev, _ptr(idx_l), _ptr(idx_next), T_fit, E, k, _ptr(W), _ptr(C),
                                 1 if accumulate else 0, _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_coselect_stats")
    return W, C


def md_place_correlated(W, R, seed_mode=MD_SEED_CONTIGUOUS, refine=True, out=None,
                        workspace=None, dev_status=None, stream=None):
    _need(W, "W", torch.int32)
    dev = W.device
    E = W.shape[0]
    if W.dim() != 2 or W.shape[1] != E:
        raise ValueError("W must be [E, E]")
    if out is None:
        out = torch.empty(E, dtype=torch.int32, device=dev)
    _need(out, "out", torch.int32, dev)
    _room(out, "out", E)
    need = int(lib().md_place_correlated_workspace_size(E, R))
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    rc = _call("md_place_correlated", dev, _ptr(W), E, R, seed_mode, 1 if refine else 0, _ptr(out),
                                   _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                   _stream(stream, dev))
    _check(rc, "md_place_correlated")
    return out


def md_place_two_level(W, R, nodes=1, seed_mode=MD_SEED_CONTIGUOUS, refine_mode=MD_REFINE_SWAPS,
                       out=None, workspace=None, dev_status=None, stream=None):
    """Placement over `nodes` nodes of R/nodes ranks (nodes=1: one level), with no
    refinement, best single swaps, or Kernighan-Lin passes."""
    _need(W, "W", torch.int32)
    dev = W.device
    E = W.shape[0]
    if W.dim() != 2 or W.shape[1] != E:
        raise ValueError("W must be [E, E]")
    if out is None:
        out = torch.empty(E, dtype=torch.int32, device=dev)
    _need(out, "out", torch.int32, dev)
    _room(out, "out", E)
    need = int(lib().md_place_two_level_workspace_size(E, R, nodes))
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    rc = _call("md_place_two_level", dev, _ptr(W), E, R, nodes, seed_mode, refine_mode, _ptr(out),
                                  _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                  _stream(stream, dev))
    _check(rc, "md_place_two_level")
    return out


def _shuffle_checks(C, E, p_next, T, dev, **outs):
    if C.dim() != 2 or C.shape[1] != E:
        raise ValueError("C must be [E, E]")
    _room(p_next, "expert_to_rank_next", E)
    for name, t in outs.items():
        _need(t, name, torch.int32, dev)
        _room(t, name, T)


def md_token_shuffle(idx_l, C, expert_to_rank_next, R, pred_rank=None, perm=None, inv=None,
                     workspace=None, dev_status=None, stream=None):
    _need(idx_l, "idx_l", torch.int32)
    dev = idx_l.device
    _need(C, "C", torch.int32, dev)
    _need(expert_to_rank_next, "expert_to_rank_next", torch.int32, dev)
    T, k = idx_l.shape
    E = C.shape[0]
    i32 = dict(dtype=torch.int32, device=dev)
    pred_rank = torch.empty(T, **i32) if pred_rank is None else pred_rank
    perm = torch.empty(T, **i32) if perm is None else perm
    inv = torch.empty(T, **i32) if inv is None else inv
    _shuffle_checks(C, E, expert_to_rank_next, T, dev, pred_rank=pred_rank, perm=perm, inv=inv)
    need = int(lib().md_token_shuffle_workspace_size(T, E, R))
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    rc = _call("md_token_shuffle", dev, _ptr(idx_l), k, _ptr(C), _ptr(expert_to_rank_next), T, E, R,
                                _ptr(pred_rank), _ptr(perm), _ptr(inv), _ptr(workspace),
                                workspace.numel(), _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_token_shuffle")
    return pred_rank, perm, inv


def md_token_shuffle_rounds(idx_l, C, expert_to_rank_next, R, pred_rank=None, perm=None,
                            inv=None, workspace=None, dev_status=None, stream=None):
    """Rounds-based capacity assignment -> (pred, perm, inv, rounds [1] device tensor)."""
    _need(idx_l, "idx_l", torch.int32)
    dev = idx_l.device
    _need(C, "C", torch.int32, dev)
    _need(expert_to_rank_next, "expert_to_rank_next", torch.int32, dev)
    T, k = idx_l.shape
    E = C.shape[0]
    i32 = dict(dtype=torch.int32, device=dev)
    pred_rank = torch.empty(T, **i32) if pred_rank is None else pred_rank
    perm = torch.empty(T, **i32) if perm is None else perm
    inv = torch.empty(T, **i32) if inv is None else inv
    _shuffle_checks(C, E, expert_to_rank_next, T, dev, pred_rank=pred_rank, perm=perm, inv=inv)
    rounds = torch.zeros(1, **i32)
    need = int(lib().md_token_shuffle_rounds_workspace_size(T, E, R))
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    rc = _call("md_token_shuffle_rounds", dev, _ptr(idx_l), k, _ptr(C), _ptr(expert_to_rank_next), T, E, R,
                                       _ptr(pred_rank), _ptr(perm), _ptr(inv), _ptr(rounds),
                                       _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                       _stream(stream, dev))
    _check(rc, "md_token_shuffle_rounds")
    return pred_rank, perm, inv, rounds


def md_coselect_pair_stats(idx_prev, idx_l, idx_next, E, T_fit=None, C2=None, accumulate=False,
                           dev_status=None, stream=None):
    """Pair counts C2[a, b, e'] (int32 view of uint32 [E, E, E])."""
    _need(idx_l, "idx_l", torch.int32)
    dev = idx_l.device
    _need(idx_prev, "idx_prev", torch.int32, dev)
    _need(idx_next, "idx_next", torch.int32, dev)
    T, k = idx_l.shape
    T_fit = T if T_fit is None else T_fit
    if C2 is None:
        C2 = torch.empty(E, E, E, dtype=torch.int32, device=dev)
    _need(C2, "C2", torch.int32, dev)
    _room(C2, "C2", E * E * E)
    if idx_prev.shape[1] != k or idx_next.shape[1] != k:
        raise ValueError("idx_prev, idx_l and idx_next differ in k")
    if min(idx_prev.shape[0], idx_next.shape[0], T) < T_fit:
        raise ValueError("fewer than T_fit rows")
    rc = _call("md_coselect_pair_stats", dev, _ptr(idx_prev), _ptr(idx_l), _ptr(idx_next), T_fit, E, k,
                                      _ptr(C2), 1 if accumulate else 0, _ptr(dev_status),
                                      _stream(stream, dev))
    _check(rc, "md_coselect_pair_stats")
    return C2


def md_token_shuffle_pair(idx_prev, idx_l, C, C2, expert_to_rank_next, R, min_obs, pred_rank=None,
                          perm=None, inv=None, use_pair=None, workspace=None, dev_status=None,
                          stream=None):
    """Pair-based shuffle prediction with single-expert fallback -> (pred, perm, inv, use_pair)."""
    _need(idx_l, "idx_l", torch.int32)
    dev = idx_l.device
    _need(idx_prev, "idx_prev", torch.int32, dev)
    _need(C, "C", torch.int32, dev)
    _need(C2, "C2", torch.int32, dev)
    _need(expert_to_rank_next, "expert_to_rank_next", torch.int32, dev)
    T, k = idx_l.shape
    E = C.shape[0]
    i32 = dict(dtype=torch.int32, device=dev)
    pred_rank = torch.empty(T, **i32) if pred_rank is None else pred_rank
    perm = torch.empty(T, **i32) if perm is None else perm
    inv = torch.empty(T, **i32) if inv is None else inv
    use_pair = torch.empty(T, **i32) if use_pair is None else use_pair
    _shuffle_checks(C, E, expert_to_rank_next, T, dev, pred_rank=pred_rank, perm=perm, inv=inv,
                    use_pair=use_pair)
    if idx_prev.shape != idx_l.shape:
        raise ValueError("idx_prev and idx_l differ in shape")
    _room(C2, "C2", E * E * E)
    need = int(lib().md_token_shuffle_pair_workspace_size(T, E, R))
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    rc = _call("md_token_shuffle_pair", dev, _ptr(idx_prev), _ptr(idx_l), k, _ptr(C), _ptr(C2),
                                     _ptr(expert_to_rank_next), T, E, R, int(min_obs),
                                     _ptr(pred_rank), _ptr(perm), _ptr(inv), _ptr(use_pair),
                                     _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                     _stream(stream, dev))
    _check(rc, "md_token_shuffle_pair")
    return pred_rank, perm, inv, use_pair


# ------------------------------------------------------- EP exchange

class md_peer_rows(ctypes.Structure):
    """One rank's exchange buffers as this rank addresses them (include/moedispatch.h)."""
    _fields_ = [("rows", ctypes.c_void_p), ("token", ctypes.c_void_p),
                ("slot_idx", ctypes.c_void_p), ("slot_w", ctypes.c_void_p),
                ("row_base", ctypes.c_int64), ("rows_cap", ctypes.c_int64)]


@dataclass
class PeerRows:
    """Buffers of one destination rank: tensors on this device, or raw device
    addresses (ints) of another GPU's memory mapped into this process."""
    rows: object
    row_base: int
    rows_cap: int
    token: object = None
    slot_idx: object = None
    slot_w: object = None


def _addr(v):
    if v is None:
        return None
    if isinstance(v, torch.Tensor):
        return v.data_ptr()
    return int(v)


def _peer_table(peers):
    arr = (md_peer_rows * len(peers))()
    for i, q in enumerate(peers):
        arr[i] = md_peer_rows(_addr(q.rows), _addr(q.token), _addr(q.slot_idx), _addr(q.slot_w),
                              int(q.row_base), int(q.rows_cap))
    return arr


def md_exchange_plan(src_rank_offsets, me):
    """(dst_row_base [R], recv_offsets [R+1]) of rank `me` from every source's
    layout rank_offsets, gathered ([R, R+1], row s = source s), on the host."""
    rows = [[int(v) for v in r] for r in src_rank_offsets.tolist()] \
        if hasattr(src_rank_offsets, "tolist") else [[int(v) for v in r] for r in src_rank_offsets]
    R = len(rows)
    if any(len(r) != R + 1 for r in rows):
        raise ValueError("src_rank_offsets must be [R, R+1]")
    flat = (ctypes.c_int64 * (R * (R + 1)))(*[v for r in rows for v in r])
    base = (ctypes.c_int64 * R)()
    recv = (ctypes.c_int64 * (R + 1))()
    _check(lib().md_exchange_plan(ctypes.cast(flat, _P), R, int(me), ctypes.cast(base, _P),
                                  ctypes.cast(recv, _P)), "md_exchange_plan")
    return list(base), list(recv)


def md_dispatch_exchange(x, topk_idx, topk_w, expert_to_rank, E, row_of_slot, rank_offsets,
                         token_base, peers, dev_status=None, stream=None):
    """Write this rank's dispatch rows (and their metadata) into the R
    destination ranks' buffers `peers` (a list of PeerRows)."""
    _need(x, "x", torch.bfloat16)
    dev = x.device
    _need(topk_idx, "topk_idx", torch.int32, dev)
    if topk_w is not None:
        _need(topk_w, "topk_w", torch.float32, dev)
    _need(expert_to_rank, "expert_to_rank", torch.int32, dev)
    _need(row_of_slot, "row_of_slot", torch.int32, dev)
    _need(rank_offsets, "rank_offsets", torch.int32, dev)
    T, H = x.shape
    k = topk_idx.shape[1]
    R = len(peers)
    _room(rank_offsets, "rank_offsets", R + 1)
    _room(row_of_slot, "row_of_slot", T * k)
    tab = _peer_table(peers)
    rc = _call("md_dispatch_exchange", dev, _ptr(x), T, H, k, _ptr(topk_idx), _ptr(topk_w),
               _ptr(expert_to_rank), E, R, _ptr(row_of_slot), _ptr(rank_offsets), int(token_base),
               ctypes.cast(tab, _P), _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_dispatch_exchange")


def md_combine_partials(y, y_row, slot_idx, slot_w, out=None, dev_status=None, stream=None):
    """Return rows of a receiving rank: z[i] = bf16(sum over carried slots, by
    ascending expert, of slot_w * y[y_row])."""
    _need(y, "y", torch.bfloat16)
    dev = y.device
    _need(y_row, "y_row", torch.int32, dev)
    _need(slot_idx, "slot_idx", torch.int32, dev)
    _need(slot_w, "slot_w", torch.float32, dev)
    n, k = y_row.shape
    H = y.shape[1]
    if slot_idx.shape != (n, k) or slot_w.shape != (n, k):
        raise ValueError("y_row, slot_idx and slot_w differ in shape")
    if out is None:
        out = torch.empty(n, H, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    _room(out, "out", n * H)
    rc = _call("md_combine_partials", dev, _ptr(y), y.shape[0], _ptr(y_row), _ptr(slot_idx),
               _ptr(slot_w), n, k, H, _ptr(out), _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_combine_partials")
    return out


def md_combine_exchange(peers, topk_idx, expert_to_rank, E, row_of_slot, rank_offsets, H,
                        out=None, dev_status=None, stream=None):
    """out[t] = bf16(fp32 sum, by ascending rank, of the return rows of t read
    from the R ranks' buffers `peers`)."""
    _need(topk_idx, "topk_idx", torch.int32)
    dev = topk_idx.device
    _need(expert_to_rank, "expert_to_rank", torch.int32, dev)
    _need(row_of_slot, "row_of_slot", torch.int32, dev)
    _need(rank_offsets, "rank_offsets", torch.int32, dev)
    T, k = topk_idx.shape
    R = len(peers)
    _room(rank_offsets, "rank_offsets", R + 1)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    _room(out, "out", T * H)
    tab = _peer_table(peers)
    rc = _call("md_combine_exchange", dev, ctypes.cast(tab, _P), T, H, k, _ptr(topk_idx),
               _ptr(expert_to_rank), E, R, _ptr(row_of_slot), _ptr(rank_offsets), _ptr(out),
               _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_combine_exchange")
    return out


# ------------------------------------------------------------ statistics

def md_rank_stats(topk_idx, E, R, expert_to_rank, hist=None, dev_status=None, stream=None):
    """hist int64 [k+1]: tokens whose experts sit on exactly D distinct ranks."""
    _need(topk_idx, "topk_idx", torch.int32)
    dev = topk_idx.device
    _need(expert_to_rank, "expert_to_rank", torch.int32, dev)
    T, k = topk_idx.shape
    hist = torch.empty(k + 1, dtype=torch.int64, device=dev) if hist is None else hist
    _need(hist, "hist", torch.int64, dev)
    _room(hist, "hist", k + 1)
    _room(expert_to_rank, "expert_to_rank", E)
    rc = _call("md_rank_stats", dev, _ptr(topk_idx), T, E, k, R, _ptr(expert_to_rank), _ptr(hist),
                             _ptr(dev_status), _stream(stream, dev))
    _check(rc, "md_rank_stats")
    return hist


def table1_row(hist):
    """Table I columns from a rank histogram: (same-rank %, ranks per token, dedup %)
    (md_table1_row on the host)."""
    h = (ctypes.c_int64 * len(hist))(*[int(v) for v in hist.tolist()])
    out = (ctypes.c_double * 3)()
    _check(lib().md_table1_row(ctypes.cast(h, _P), len(hist) - 1, ctypes.cast(out, _P)),
           "md_table1_row")
    return out[0], out[1], out[2]


def md_successor_share(C, W, stream=None):
    """(num, den) int32 views of uint32 [E]: max_e' C[e, e'] and W[e, e]."""
    _need(C, "C", torch.int32)
    dev = C.device
    _need(W, "W", torch.int32, dev)
    E = C.shape[0]
    if C.shape != (E, E) or W.shape != (E, E):
        raise ValueError("C and W must be [E, E]")
    num = torch.empty(E, dtype=torch.int32, device=dev)
    den = torch.empty(E, dtype=torch.int32, device=dev)
    rc = _call("md_successor_share", dev, _ptr(C), _ptr(W), E, _ptr(num), _ptr(den), _stream(stream, dev))
    _check(rc, "md_successor_share")
    return num, den


def md_count_sums(x, y, stream=None):
    """Exact (sx, sy, sxx, syy, sxy) of two count tables (int32 views of uint32)."""
    _need(x, "x", torch.int32)
    dev = x.device
    _need(y, "y", torch.int32, dev)
    if x.numel() != y.numel():
        raise MoeDispatchError("md_count_sums: tables differ in size")
    out = torch.empty(10, dtype=torch.int64, device=dev)
    rc = _call("md_count_sums", dev, _ptr(x), _ptr(y), x.numel(), _ptr(out), _stream(stream, dev))
    _check(rc, "md_count_sums")
    w = [v & (2 ** 64 - 1) for v in out.cpu().tolist()]
    return tuple(w[2 * i] | (w[2 * i + 1] << 64) for i in range(5))


def pearson_from_sums(n, sums):
    """Pearson correlation from the exact sums of md_count_sums (md_pearson_from_sums
    on the host); NaN when a table has zero variance."""
    words = []
    for v in sums:
        v = int(v)
        words += [v & (2 ** 64 - 1), (v >> 64) & (2 ** 64 - 1)]
    c = (ctypes.c_uint64 * 10)(*words)
    r = ctypes.c_double()
    rc = lib().md_pearson_from_sums(ctypes.cast(c, _P), int(n), ctypes.byref(r))
    if rc == MD_ERR_DATA:
        return float("nan")
    _check(rc, "md_pearson_from_sums")
    return r.value


def md_set_test_hooks(poll_limit=0, layout_skip_tile=-1, expand_skip_unit=-1):
    """Fault injection for tests: make a bounded device-side wait run out."""
    lib().md_set_test_hooks(int(poll_limit), int(layout_skip_tile), int(expand_skip_unit))
