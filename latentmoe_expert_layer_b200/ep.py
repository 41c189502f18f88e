"""Expert-parallel data movement of the LatentMoE layer across ranks (one process per GPU).

The "Nemotron 3 Super" notes (section 3.2) motivate the latent projection by the all-to-all routing
traffic of distributed MoE, which grows with the dimension of the dispatched vectors times K: a
LatentMoE dispatches the l-dimensional latent h = W_down x instead of x, d / l times fewer bytes.

Each of G ranks owns a contiguous range of N / G experts.  A forward on rank r, for its own tokens:

  1. route     idx, gate (router in d) and h = W_down x, locally;
  2. dispatch  every assignment (t, k) goes to the owner of idx[t, k]: its latent row h[t], its expert
               id and its gate travel in one all-to-all each, in (token, slot) order per destination;
  3. experts   the owner groups the received rows by local expert (stably, in arrival order) and runs
               its experts on them, the gate folded into the output;
  4. return    the outputs travel back to their source rank (the reverse all-to-all);
  5. combine   z[t] = sum_k o[t, k] in slot order, then y = W_up z + shared expert (x), locally.

This module is the data movement only.  The compute steps are callables (route, experts, output), so
the same plan runs with the library's kernels on GPUs over NCCL or, in the tests, with any reference
implementation on CPU ranks over gloo.  Collectives are the torch.distributed ones; the exchanged
sizes are agreed with one all-to-all of per-destination counts (its result is read on the host).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["ExpertPartition", "DispatchPlan", "plan_dispatch", "group_by_local_expert", "dispatch_bytes",
           "ep_forward"]


@dataclasses.dataclass(frozen=True)
class ExpertPartition:
    """Contiguous expert ownership: rank r owns experts [r * per_rank, (r + 1) * per_rank)."""
    n_experts: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.n_experts % self.world:
            raise ValueError("the expert count must be a multiple of the number of ranks")

    @property
    def per_rank(self) -> int:
        return self.n_experts // self.world

    def owner(self, expert: torch.Tensor) -> torch.Tensor:
        return torch.div(expert, self.per_rank, rounding_mode="floor")

    def first(self, rank: int) -> int:
        return rank * self.per_rank


@dataclasses.dataclass
class DispatchPlan:
    order: torch.Tensor        # [T*K] assignments (t*K + k) in send order: by destination, then (t, k)
    send_counts: torch.Tensor  # [G] assignments sent to each rank


def plan_dispatch(idx: torch.Tensor, part: ExpertPartition) -> DispatchPlan:
    """Send order of the (token, slot) assignments: grouped by owning rank, (token, slot) order
    within a rank (a stable sort of the owners)."""
    flat = idx.reshape(-1).to(torch.int64)
    dest = part.owner(flat)
    _, order = torch.sort(dest, stable=True)
    return DispatchPlan(order, torch.bincount(dest, minlength=part.world))


def group_by_local_expert(expert: torch.Tensor, first: int, per_rank: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Stable grouping of received assignments by local expert: (order, rows per local expert)."""
    local = expert.to(torch.int64) - first
    if local.numel() and (int(local.min()) < 0 or int(local.max()) >= per_rank):
        raise ValueError("an assignment reached a rank that does not own its expert")
    _, order = torch.sort(local, stable=True)
    return order, torch.bincount(local, minlength=per_rank)


def dispatch_bytes(tokens: int, top_k: int, width: int, elem_bytes: int = 2) -> int:
    """Bytes of dispatched rows for `tokens` tokens: one row of `width` elements per assignment
    (the same again on the way back)."""
    return tokens * top_k * width * elem_bytes


def _exchange(send: torch.Tensor, send_counts: list, recv_counts: list, group) -> torch.Tensor:
    out = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(out, send.contiguous(), recv_counts, send_counts, group=group)
    return out


def ep_forward(x: torch.Tensor, part: ExpertPartition,
               route: Callable[[torch.Tensor], Tuple[torch.Tensor, torch.Tensor, torch.Tensor]],
               experts: Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor],
               output: Callable[[torch.Tensor, torch.Tensor], torch.Tensor],
               group: Optional["dist.ProcessGroup"] = None):
    """One expert-parallel forward of this rank's tokens x [T, d].

    route(x)                         -> idx [T, K] (global expert ids), gate [T, K], h [T, l]
    experts(rows, counts, gates)     -> o [R, l]: rows grouped by local expert (counts per local
                                        expert, in order), outputs already multiplied by the gates
    output(z, x)                     -> y [T, d] from the latent sum z [T, l]
    Every rank calls this at the same point (it runs five all-to-alls).  Returns (y, idx, gate)."""
    rank = dist.get_rank(group)
    idx, gate, h = route(x)
    t, k = idx.shape
    plan = plan_dispatch(idx, part)
    send_counts = plan.send_counts.tolist()
    recv_counts_t = torch.empty(part.world, dtype=torch.int64, device=plan.send_counts.device)
    dist.all_to_all_single(recv_counts_t, plan.send_counts.to(torch.int64), group=group)
    recv_counts = recv_counts_t.tolist()

    tok = torch.div(plan.order, k, rounding_mode="floor")
    rows = _exchange(h[tok], send_counts, recv_counts, group)
    eids = _exchange(idx.reshape(-1)[plan.order].to(torch.int64), send_counts, recv_counts, group)
    gates = _exchange(gate.reshape(-1)[plan.order], send_counts, recv_counts, group)

    gorder, counts = group_by_local_expert(eids, part.first(rank), part.per_rank)
    o_grouped = experts(rows[gorder], counts, gates[gorder])
    o_arrival = torch.empty_like(o_grouped)
    o_arrival[gorder] = o_grouped
    back = _exchange(o_arrival, recv_counts, send_counts, group)   # the reverse exchange
    o = torch.empty((t * k, h.shape[1]), dtype=back.dtype, device=back.device)
    o[plan.order] = back
    o = o.reshape(t, k, h.shape[1])
    z = o[:, 0].clone()
    for s in range(1, k):           # slot order
        z += o[:, s]
    return output(z, x), idx, gate
