"""Expert parallelism: the exchange plan (host logic).

With R ranks, expert e lives on rank e // (N / R).  Every rank routes its own
tokens; a dispatch (t, s) of rank r goes to the owner of its expert.  The
capacity of an expert counts the dispatches of all ranks in one global order:
rank 0's tokens first, then rank 1's, and so on, each in token order.  The
expert-parallel layer therefore computes exactly the single-GPU layer of
"Mixture of Experts MoE: how sparse activation saves compute" (§3.5, §3.6,
§3.8) on the ranks' batches laid end to end.  The tutorial names the
all-to-all dispatch and combine as the multi-device cost of this layout.

Per step, each rank groups its own dispatches by expert with no capacity
(moe_permute with capacity 0), so its dispatches to expert e are a contiguous
run of counts[e] rows in token order, and exchanges the per-expert counts
(exchange_counts, one all-gather of R x N integers).  From the R x N counts,
plan() derives for every rank, with no further communication:

  kept[e]        my dispatches to e that fit the capacity: the first kept[e]
                 of my run for e (the ranks before me take their share first)
  local_offsets  my grouped layout of kept rows, exclusive prefix of kept
  send_base[e]   row of the owner's receive buffer where my kept rows for e
                 start; my j-th kept dispatch to e lands at send_base[e] + j
  send_counts[o] rows I send to rank o (its experts' kept rows, expert order)
  recv_offsets   my receive buffer grouped by my local experts, then by
                 source rank, then by the source's token order
  recv_src_base[el][r]  row of my receive buffer where source r's rows for my
                 local expert el start (for putting results back)
  recv_counts[r] rows I receive from rank r

The owner computes each received row's expert output in place; the results
go back to the source rank's local grouped row local_offsets[e] + j, where the
source's combine (moe_combine semantics, weights not renormalised over
drops) finishes the layer.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class EpPlan:
    rank: int
    world: int
    experts_per_rank: int
    kept: np.ndarray           # [N] int32
    local_offsets: np.ndarray  # [N + 1]
    send_base: np.ndarray      # [N]
    send_counts: np.ndarray    # [R]
    recv_offsets: np.ndarray   # [E_loc + 1]
    recv_src_base: np.ndarray  # [E_loc][R]
    recv_counts: np.ndarray    # [R]
    overflow: np.ndarray       # [N] dropped dispatches of all ranks per expert

    @property
    def recv_rows(self) -> int:
        return int(self.recv_offsets[-1])

    def owner(self, e: int) -> int:
        return e // self.experts_per_rank


def owner_of(e: int, N: int, world: int) -> int:
    """Rank that holds expert e: N / world consecutive experts per rank."""
    return e // (N // world)


def plan(counts_all, capacity: int, rank: int) -> EpPlan:
    """The exchange plan of `rank` from every rank's per-expert dispatch
    counts counts_all [R][N] (before capacity) and the per-expert capacity C
    (0 = unlimited), computed by the library's host-only moe_ep_plan.  Every
    rank derives the same global picture from the same counts."""
    from . import moe_ep_plan
    c = np.asarray(counts_all)
    if c.ndim != 2:
        raise ValueError("counts_all must be [world][N]")
    R, N = c.shape
    if R < 1 or N % R != 0 or not 0 <= rank < R:
        raise ValueError(f"{N} experts do not split over {R} ranks, or rank {rank} is out of range")
    if capacity < 0 or (c < 0).any():
        raise ValueError("negative capacity or count")
    p = moe_ep_plan(c, capacity, rank)
    return EpPlan(rank, R, N // R, p["kept"], p["local_offsets"], p["send_base"],
                  p["send_counts"], p["recv_offsets"], p["recv_src_base"], p["recv_counts"],
                  p["overflow"])


def exchange_counts(counts_local, group=None):
    """All ranks' per-expert dispatch counts [R][N] from this rank's [N]
    (torch.distributed all-gather; NCCL on GPUs, gloo on CPU)."""
    import torch
    import torch.distributed as dist
    t = torch.as_tensor(counts_local).to(torch.int64).reshape(-1)
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t, group=group)
    return torch.stack(parts).cpu().numpy()
