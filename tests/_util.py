"""Shared helpers for the parity tests (marshalling only, no arithmetic of the path)."""
import numpy as np
import torch

import oracle
from combine_warp_top_router_b200 import synth

DEV = "cuda"


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 numpy bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray, device=DEV) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16).copy()).view(torch.bfloat16).to(device)


def i32(a, device=DEV) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def f32(a, device=DEV) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)


def logits_for(name, T, seed=0, R=None):
    """Layer-l (and l+1 when the workload has one) logits on the CPU."""
    w = synth.make_workload(name, seed=seed, device="cpu", T=T, R=R, with_rows=False)
    return w


def oracle_route(logits_cpu: torch.Tensor, k, mode=0):
    return oracle.route_topk(logits_cpu.numpy(), k, mode)


def shuffled_placement(E, R, seed):
    p = (np.arange(E) // (E // R)).astype(np.int32)
    return np.random.default_rng(seed).permutation(p).astype(np.int32)
