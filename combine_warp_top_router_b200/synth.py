"""Seeded synthetic inputs shaped like the source pages' workloads.

This module only draws random numbers and lays them out.  It holds none of the
dispatch / combine arithmetic: no top-k, no layout, no combine.  The test suite
(for both the CUDA library and the oracle) and ``bench.py`` take their inputs
from here, so both sides of every parity check see identical bytes.

Every tensor has its own generator, seeded from ``(seed, tag)``, so the value of
one tensor never depends on which other tensors were drawn before it.

Shapes follow the pages:
  * "DODOCO: MoE AlltoAll Traffic Matrices on Real Text", Models table and Setup:
    (E, k, hidden) = (64, 6, 2048), (128, 8, 2048), (256, 8, 2048); 16 ranks that
    each route 4096 tokens; contiguous expert placement.
  * "Expert Coupling in MoE Pretraining", Model Configuration: d_model 4096,
    128 experts, top-2 / top-6; Within-layer correlation: a few expert pairs
    carry a large share of tokens; Cross-layer correlation: a layer-l expert
    sends most of its tokens to one layer-l+1 expert.
The real routing traces behind those pages are not available, so the
correlated structure is planted: boosted expert groups drawn Zipf(1.1) per
token, boosted pairs, and a boosted successor of the previous layer's top-1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# tags: one per independent random tensor
_T_LOGITS, _T_LOGITS_NEXT, _T_X, _T_Y = 1, 2, 3, 4
_T_GROUPS, _T_ZIPF, _T_PAIRS, _T_PAIR_PICK, _T_PAIR_ON = 5, 6, 7, 8, 9
_T_SUCC, _T_SKEW, _T_GROUPS_NEXT, _T_ZIPF_NEXT = 10, 11, 12, 13
_T_LOGITS_PREV, _T_GROUPS_PREV, _T_ZIPF_PREV, _T_SUCC_PAIR = 14, 15, 16, 17


def generator(seed: int, tag: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 0x9E3779B1 + int(tag) * 0x85EBCA77 + 0x2545F491) % (1 << 62))
    return g


def normal_f32(rows: int, cols: int, seed: int, tag: int, device="cpu") -> torch.Tensor:
    return torch.randn(rows, cols, generator=generator(seed, tag, device), device=device,
                       dtype=torch.float32)


def normal_bf16(rows: int, cols: int, seed: int, tag: int, device="cpu",
                chunk_rows: int = 1 << 16) -> torch.Tensor:
    """N(0,1) rounded to bf16 (round to nearest even), drawn in row chunks."""
    g = generator(seed, tag, device)
    out = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn(r1 - r0, cols, generator=g, device=device,
                                 dtype=torch.float32).to(torch.bfloat16)
    return out


def contiguous_placement(E: int, R: int, device="cpu") -> torch.Tensor:
    """Rank r holds experts r*E/R .. (r+1)*E/R - 1 (DODOCO, Setup)."""
    return (torch.arange(E, dtype=torch.int32, device=device) // (E // R)).to(torch.int32)


def _zipf_draw(n: int, n_items: int, s: float, g: torch.Generator, device) -> torch.Tensor:
    """n draws of an item index 0..n_items-1 with P(i) proportional to (i+1)^-s."""
    probs = torch.arange(1, n_items + 1, dtype=torch.float64, device=device).pow(-s)
    probs = (probs / probs.sum()).to(torch.float32)
    return torch.multinomial(probs, n, replacement=True, generator=g)


def group_boost_logits(T: int, E: int, group_size: int, boost: float, seed: int,
                       tag_noise: int, tag_groups: int, tag_zipf: int, zipf_s: float = 1.1,
                       device="cpu") -> torch.Tensor:
    """N(0,1) logits plus `boost` on every expert of one group per token.

    Groups: a seeded random partition of the E experts into E/group_size groups.
    Each token draws its group Zipf(zipf_s) over the groups' rank order.
    """
    logits = normal_f32(T, E, seed, tag_noise, device)
    n_groups = E // group_size
    perm = torch.randperm(E, generator=generator(seed, tag_groups, device), device=device)
    groups = perm.view(n_groups, group_size)
    gid = _zipf_draw(T, n_groups, zipf_s, generator(seed, tag_zipf, device), device)
    rows = torch.arange(T, device=device).unsqueeze(1).expand(T, group_size)
    logits[rows, groups[gid]] += boost
    return logits


def pair_boost_logits(T: int, E: int, n_pairs: int, boost: float, frac: float, seed: int,
                      device="cpu") -> torch.Tensor:
    """N(0,1) logits; a fraction `frac` of tokens gets `boost` on both experts
    of one uniformly chosen pair out of `n_pairs` disjoint pairs."""
    logits = normal_f32(T, E, seed, _T_LOGITS, device)
    perm = torch.randperm(E, generator=generator(seed, _T_PAIRS, device), device=device)
    pairs = perm[: 2 * n_pairs].view(n_pairs, 2)
    pick = torch.randint(0, n_pairs, (T,), generator=generator(seed, _T_PAIR_PICK, device),
                         device=device)
    on = torch.rand(T, generator=generator(seed, _T_PAIR_ON, device), device=device) < frac
    rows = torch.nonzero(on).squeeze(1)
    for c in range(2):
        logits[rows, pairs[pick[rows], c]] += boost
    return logits


def load_skew_bias(E: int, ratio: float, seed: int, device="cpu") -> torch.Tensor:
    """b_e = ln(ratio) * (1 - q_e / (E - 1)), q a seeded permutation of 0..E-1:
    a ratio:1 max/min prior on expert popularity."""
    q = torch.randperm(E, generator=generator(seed, _T_SKEW, device), device=device)
    return (math.log(ratio) * (1.0 - q.to(torch.float32) / (E - 1))).to(torch.float32)


def successor_map(E: int, seed: int, device="cpu") -> torch.Tensor:
    """A fixed random map expert -> layer-l+1 successor expert."""
    return torch.randint(0, E, (E,), generator=generator(seed, _T_SUCC, device), device=device)


def boost_successor(next_logits: torch.Tensor, prev_logits: torch.Tensor, succ: torch.Tensor,
                    boost: float) -> torch.Tensor:
    """Add `boost` at succ[first argmax of the previous layer's logits] per token.
    (torch.argmax returns the first maximal index.)"""
    top1 = torch.argmax(prev_logits, dim=1)
    out = next_logits.clone()
    out[torch.arange(out.shape[0], device=out.device), succ[top1]] += boost
    return out


def pair_successor_map(E: int, seed: int, device="cpu") -> torch.Tensor:
    """A fixed random map (expert at l-1, expert at l) -> layer-l+1 expert, [E, E]."""
    return torch.randint(0, E, (E, E), generator=generator(seed, _T_SUCC_PAIR, device),
                         device=device)


def boost_pair_successor(next_logits: torch.Tensor, prev2_logits: torch.Tensor,
                         prev_logits: torch.Tensor, succ2: torch.Tensor,
                         boost: float) -> torch.Tensor:
    """Add `boost` at succ2[first argmax at l-1, first argmax at l] per token."""
    a = torch.argmax(prev2_logits, dim=1)
    b = torch.argmax(prev_logits, dim=1)
    out = next_logits.clone()
    out[torch.arange(out.shape[0], device=out.device), succ2[a, b]] += boost
    return out


@dataclass
class Workload:
    """One synthetic problem.  Tensors live on `device`."""
    name: str
    T: int
    H: int
    E: int
    k: int
    R: int
    mode: int                      # 0 conventional, 1 dedup
    logits: torch.Tensor           # float32 [T, E]
    x: torch.Tensor | None         # bf16 [T, H]
    y: torch.Tensor | None         # bf16 [T*k, H] expert outputs, conventional row order
    expert_to_rank: torch.Tensor   # int32 [E]
    logits_next: torch.Tensor | None = None
    fit_tokens: int = 0
    logits_prev: torch.Tensor | None = None  # layer l-1, three-layer workloads only
    extra: dict = field(default_factory=dict)


# The five workloads.  Each entry: (T, H, E, k, R, mode, description).
SPECS = {
    "iid_e64_k6": dict(T=4096, H=2048, E=64, k=6, R=16, mode=0,
                       desc="T=4096 H=2048 E=64 top-6 R=16, iid N(0,1) logits, contiguous, conventional"),
    "zipf_pairs_e128_k8": dict(T=65536, H=2048, E=128, k=8, R=16, mode=1,
                               desc="T=65536 H=2048 E=128 top-8 R=16, +3.0 on one of 64 expert pairs "
                                    "drawn Zipf(1.1) per token, contiguous, dedup"),
    "boost_pairs_e128_k2": dict(T=65536, H=4096, E=128, k=2, R=8, mode=1,
                                desc="T=65536 H=4096 E=128 top-2 R=8 (or 32), +3.5 on one of 64 pairs for "
                                     "40% of tokens, correlated placement fitted on 4096 tokens, dedup"),
    "two_layer_e128_k6": dict(T=65536, H=2048, E=128, k=6, R=16, mode=1,
                              desc="T=65536 H=2048 E=128 top-6 R=16, two layers, layer l+1 boosted on a "
                                   "fixed successor of the layer-l top-1, token shuffle, dedup"),
    "three_layer_e128_k6": dict(T=65536, H=2048, E=128, k=6, R=16, mode=1,
                                desc="T=65536 H=2048 E=128 top-6 R=16, three layers: layer l boosted "
                                     "on a fixed successor of the layer-(l-1) top-1, layer l+1 on a "
                                     "fixed successor of the (l-1, l) top-1 pair; pair-based shuffle"),
    "full_e256_k8": dict(T=262144, H=2048, E=256, k=8, R=64, mode=1,
                         desc="T=262144 H=2048 E=256 top-8 R=64, +3.0 on one of 64 groups of 4 drawn "
                              "Zipf(1.1), x4 load skew, full pipeline, dedup"),
}


def make_workload(name: str, seed: int = 0, device="cpu", T: int | None = None,
                  H: int | None = None, R: int | None = None, with_rows: bool = True,
                  mode: int | None = None) -> Workload:
    """Build workload `name`; T, H, R and mode may be overridden (smaller tests)."""
    s = dict(SPECS[name])
    T = s["T"] if T is None else T
    H = s["H"] if H is None else H
    R = s["R"] if R is None else R
    E, k = s["E"], s["k"]
    mode = s["mode"] if mode is None else mode
    nxt = None
    fit = 0
    if name == "iid_e64_k6":
        logits = normal_f32(T, E, seed, _T_LOGITS, device)
    elif name == "zipf_pairs_e128_k8":
        logits = group_boost_logits(T, E, 2, 3.0, seed, _T_LOGITS, _T_GROUPS, _T_ZIPF, device=device)
    elif name == "boost_pairs_e128_k2":
        logits = pair_boost_logits(T, E, 64, 3.5, 0.40, seed, device=device)
        fit = min(T, 4096)
    elif name == "two_layer_e128_k6":
        logits = group_boost_logits(T, E, 2, 3.0, seed, _T_LOGITS, _T_GROUPS, _T_ZIPF, device=device)
        fresh = group_boost_logits(T, E, 2, 3.0, seed, _T_LOGITS_NEXT, _T_GROUPS_NEXT, _T_ZIPF_NEXT,
                                   device=device)
        nxt = boost_successor(fresh, logits, successor_map(E, seed, device), 3.0)
        fit = min(T, 4096)
    elif name == "three_layer_e128_k6":
        prev = group_boost_logits(T, E, 2, 3.0, seed, _T_LOGITS_PREV, _T_GROUPS_PREV, _T_ZIPF_PREV,
                                  device=device)
        fresh = group_boost_logits(T, E, 2, 3.0, seed, _T_LOGITS, _T_GROUPS, _T_ZIPF, device=device)
        logits = boost_successor(fresh, prev, successor_map(E, seed, device), 3.0)
        fresh = group_boost_logits(T, E, 2, 3.0, seed, _T_LOGITS_NEXT, _T_GROUPS_NEXT, _T_ZIPF_NEXT,
                                   device=device)
        nxt = boost_pair_successor(fresh, prev, logits, pair_successor_map(E, seed, device), 3.0)
        fit = min(T, 4096)
    elif name == "full_e256_k8":
        bias = load_skew_bias(E, 4.0, seed, device)
        logits = group_boost_logits(T, E, 4, 3.0, seed, _T_LOGITS, _T_GROUPS, _T_ZIPF,
                                    device=device) + bias
        fresh = group_boost_logits(T, E, 4, 3.0, seed, _T_LOGITS_NEXT, _T_GROUPS_NEXT, _T_ZIPF_NEXT,
                                   device=device) + bias
        nxt = boost_successor(fresh, logits, successor_map(E, seed, device), 3.0)
        fit = T
    else:
        raise KeyError(name)
    x = normal_bf16(T, H, seed, _T_X, device) if with_rows else None
    y = normal_bf16(T * k, H, seed, _T_Y, device) if with_rows else None
    return Workload(name=name, T=T, H=H, E=E, k=k, R=R, mode=mode, logits=logits.contiguous(),
                    x=x, y=y, expert_to_rank=contiguous_placement(E, R, device),
                    logits_next=None if nxt is None else nxt.contiguous(), fit_tokens=fit,
                    logits_prev=prev.contiguous() if name == "three_layer_e128_k6" else None)
