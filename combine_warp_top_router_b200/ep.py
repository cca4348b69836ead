"""Expert-parallel exchange across GPUs, one process per GPU (plumbing).

"Expert Coupling in MoE Pretraining", The Communication Bottleneck: each MoE
layer runs a dispatch and a combine all-to-all.  Here they are two kernels of
libmoedispatch that write and read the other ranks' buffers directly
(md_dispatch_exchange, md_combine_exchange), around the receiving rank's
md_combine_partials.  This module only moves arguments and runs the
torch.distributed steps around them:

  1. every rank lays out its own tokens (md_dispatch_layout);
  2. ``gather_rank_offsets``: one all-gather of the R+1 rank offsets of every
     rank's layout (the count exchange; R+1 int32 per rank);
  3. ``md_exchange_plan`` (library, on the host): where each rank's block
     starts in every destination, and how many rows this rank receives;
  4. ``ExchangeBuffers``: receive and return buffers that every rank can
     address -- torch symmetric memory, whose peer pointers map the other
     GPUs' buffers over NVLink -- or plain local tensors when the group has
     one rank (or for tests that play every rank on one GPU);
  5. ``dispatch``: the rows into the destinations, then a barrier; the
     receiver's experts and ``md_combine_partials``; ``combine``: a barrier,
     then the return rows read back and summed.

No step here computes anything of the method: the counts, offsets, rows and
sums all come from the library.  The data path has no library collective
and no multicast.
"""
from __future__ import annotations

import torch

from . import binding as md


def gather_rank_offsets(rank_offsets: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's layout rank_offsets (int32 [R+1]) -> int32
    [world, R+1], row s from rank s.  A single process returns its own row."""
    import torch.distributed as dist
    ro = rank_offsets.to(torch.int32).contiguous().view(1, -1)
    if not dist.is_available() or not dist.is_initialized():
        return ro.clone()
    world = dist.get_world_size(group)
    out = torch.empty(world, ro.shape[1], dtype=torch.int32, device=ro.device)
    dist.all_gather_into_tensor(out, ro, group=group)
    return out


def plan(gathered_rank_offsets: torch.Tensor, me: int):
    """md_exchange_plan on the gathered offsets -> (dst_row_base, recv_offsets)."""
    return md.md_exchange_plan(gathered_rank_offsets.cpu().to(torch.int64), me)


class ExchangeBuffers:
    """One rank's receive buffers (dispatch rows and their metadata) and return
    buffer (combine rows), addressable by every rank of the group.

    rows_cap: the most rows this rank can receive in one step (a dedup
    dispatch sends a token at most one row per rank, so the group's token
    count bounds it)."""

    def __init__(self, rows_cap: int, H: int, k: int, device, group=None, symmetric=None):
        import torch.distributed as dist
        self.rows_cap, self.H, self.k = int(rows_cap), int(H), int(k)
        self.group = group
        on = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if on else 1
        self.rank = dist.get_rank(group) if on else 0
        # symmetric memory whenever other ranks must reach these buffers (and
        # on request, e.g. to exercise it with a one-rank group)
        self.symmetric = (self.world > 1) if symmetric is None else bool(symmetric)
        shapes = {"rows": ((self.rows_cap, H), torch.bfloat16), "token": ((self.rows_cap,), torch.int32),
                  "slot_idx": ((self.rows_cap, k), torch.int32),
                  "slot_w": ((self.rows_cap, k), torch.float32),
                  "ret": ((self.rows_cap, H), torch.bfloat16)}
        self.local = {}
        self.ptrs = {}
        if self.symmetric:
            import torch.distributed._symmetric_memory as symm
            for name, (shape, dtype) in shapes.items():
                t = symm.empty(*shape, dtype=dtype, device=device)
                h = symm.rendezvous(t, group if group is not None else dist.group.WORLD)
                self.local[name] = t
                self.ptrs[name] = list(h.buffer_ptrs)
        else:
            for name, (shape, dtype) in shapes.items():
                t = torch.empty(*shape, dtype=dtype, device=device)
                self.local[name] = t
                self.ptrs[name] = [t.data_ptr()]

    def peers(self, dst_row_base, caps, which="dispatch"):
        """PeerRows of every rank d for this source: its block starts at
        dst_row_base[d]; `caps` holds each rank's rows_cap."""
        out = []
        for d in range(len(dst_row_base)):
            if which == "dispatch":
                out.append(md.PeerRows(rows=self.ptrs["rows"][d], token=self.ptrs["token"][d],
                                       slot_idx=self.ptrs["slot_idx"][d],
                                       slot_w=self.ptrs["slot_w"][d],
                                       row_base=dst_row_base[d], rows_cap=caps[d]))
            else:
                out.append(md.PeerRows(rows=self.ptrs["ret"][d], row_base=dst_row_base[d],
                                       rows_cap=caps[d]))
        return out


def dispatch(x, topk_idx, topk_w, expert_to_rank, E, bufs: ExchangeBuffers, dev_status=None):
    """This rank's side of the dispatch all-to-all.

    x bf16 [T, H] and topk_idx / topk_w [T, k] are this rank's T tokens (the
    group's tokens are the ranks' blocks in rank order, so token t here is
    global token rank*T + t).  Lays the tokens out (dedup), exchanges the
    layout offsets, writes every row into its destination rank's buffers and
    waits for the group.  Returns (layout, rows received): bufs.local["rows"]
    [:rows], ["token"], ["slot_idx"], ["slot_w"] then hold what this rank's
    experts must process, in (source rank, token) order."""
    R, me = bufs.world, bufs.rank
    T = x.shape[0]
    L = md.md_dispatch_layout(topk_idx, E, R, expert_to_rank, md.MD_DEDUP, dev_status=dev_status)
    gathered = gather_rank_offsets(L.rank_offsets, bufs.group)
    base, recv = plan(gathered, me)
    md.md_dispatch_exchange(x, topk_idx, topk_w, expert_to_rank, E, L.row_of_slot, L.rank_offsets,
                            me * T, bufs.peers(base, [bufs.rows_cap] * R), dev_status=dev_status)
    L.exchange_base = base  # where this rank's blocks sit on every destination
    barrier(bufs.group)
    return L, int(recv[R])


def combine(L, topk_idx, expert_to_rank, E, bufs: ExchangeBuffers, out=None, dev_status=None):
    """This rank's side of the combine all-to-all: once every rank has written
    its return rows (bufs.local["ret"], one per received row, e.g. with
    md_combine_partials) and the group has met, read the return rows of this
    rank's tokens from their ranks and sum them."""
    barrier(bufs.group)
    R = bufs.world
    return md.md_combine_exchange(bufs.peers(L.exchange_base, [bufs.rows_cap] * R, which="combine"),
                                  topk_idx, expert_to_rank, E, L.row_of_slot, L.rank_offsets,
                                  bufs.H, out=out, dev_status=dev_status)


def barrier(group=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier(group=group)
