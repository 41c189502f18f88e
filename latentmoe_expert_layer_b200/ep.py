"""Expert-parallel data movement of the LatentMoE layer across ranks (one process per GPU).

The "Nemotron 3 Super" notes (section 3.2) motivate the latent projection by the all-to-all routing
traffic of distributed MoE, which grows with the dimension of the dispatched vectors times K: a
LatentMoE dispatches the l-dimensional latent h = W_down x instead of x, d / l times fewer bytes.

Each of G ranks owns a contiguous range of N / G experts.  A forward on rank r, for its own tokens:

  1. route     idx, gate (router in d) and h = W_down x, locally;
  2. dispatch  a token's latent row h[t] travels ONCE to every rank that owns at least one of its K
               experts (one row per (token, destination) pair, not per assignment); beside it go the
               assignments themselves: (pair index, expert id) and the gate, in (token, slot) order;
  3. experts   the owner expands the pairs to assignment rows, groups them by local expert (stably,
               in arrival order) and runs its experts, the gate folded into the output;
  4. reduce    the owner sums the outputs of each (token, source rank) pair in slot order, so one
               partial latent sum per pair goes back: at most min(K, G) rows of l per token;
  5. return    the partial sums travel back to their source rank (the reverse all-to-all);
  6. combine   z[t] = sum of the partial sums in ascending owner-rank order, then
               y = W_up z + shared expert (x), locally.

The sum in z is the same set of K gated expert outputs as the single-GPU layer's slot-order sum,
grouped by owner rank first; the two differ only in floating-point rounding.

Two drivers of the same plan:
  ep_forward          the compute steps are callables (route, experts, output), so the plan runs with
                      any implementation; the tests run it on CPU ranks over gloo with the oracle;
  ep_forward_library  the compute steps are the library's lmoe_ep_dispatch / lmoe_ep_experts /
                      lmoe_ep_combine on a layer created with ep_world = G (its plan is built on the
                      device), and the exchanges are all-to-alls of the process group (NCCL on GPUs).
Collectives are the torch.distributed ones.  The exchanged sizes are agreed with one all-to-all of
per-destination counts, whose result is the only value read back on the host (the split sizes of
the other all-to-alls).  Partial sums travel at no less than fp32.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["ExpertPartition", "DispatchPlan", "plan_dispatch", "group_by_local_expert", "dispatch_bytes",
           "exchange_bytes", "reduce_pairs", "ep_forward", "ep_forward_library"]


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
    """Send order of one rank's routing, grouped by destination rank.

    pairs: the (token, destination) pairs, sorted by (destination, token); one latent row each.
    assignments: the (token, slot) assignments t*K + k, sorted by (destination, token, slot); the
    pairs of one destination are numbered from 0 in that destination's segment."""
    pair_tok: torch.Tensor       # [P] token of each pair, in send order
    pair_counts: torch.Tensor    # [G] pairs (= latent rows) sent to each rank
    order: torch.Tensor          # [T*K] assignments in send order
    assign_pair: torch.Tensor    # [T*K] pair index of each sent assignment, within its destination
    send_counts: torch.Tensor    # [G] assignments sent to each rank


def _exclusive_cumsum(c: torch.Tensor) -> torch.Tensor:
    return torch.cumsum(c, 0) - c


def plan_dispatch(idx: torch.Tensor, part: ExpertPartition) -> DispatchPlan:
    """Pairs and assignments of idx [T, K] in send order (a stable sort of the owners keeps the
    (token, slot) order inside each destination)."""
    t, k = idx.shape
    flat = idx.reshape(-1).to(torch.int64)
    dest = part.owner(flat)
    _, order = torch.sort(dest, stable=True)
    dest_s = dest[order]
    tok_s = torch.div(order, max(k, 1), rounding_mode="floor")
    key = dest_s * max(t, 1) + tok_s                       # nondecreasing along the send order
    new = torch.ones_like(key, dtype=torch.bool)
    if key.numel() > 1:
        new[1:] = key[1:] != key[:-1]
    pair_global = torch.cumsum(new.to(torch.int64), 0) - 1
    pair_dest = dest_s[new]
    pair_counts = torch.bincount(pair_dest, minlength=part.world)
    assign_pair = pair_global - _exclusive_cumsum(pair_counts)[dest_s]
    return DispatchPlan(tok_s[new], pair_counts, order, assign_pair,
                        torch.bincount(dest, minlength=part.world))


def group_by_local_expert(expert: torch.Tensor, first: int, per_rank: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Stable grouping of received assignments by local expert: (order, rows per local expert)."""
    local = expert.to(torch.int64) - first
    if local.numel() and (int(local.min()) < 0 or int(local.max()) >= per_rank):
        raise ValueError("an assignment reached a rank that does not own its expert")
    _, order = torch.sort(local, stable=True)
    return order, torch.bincount(local, minlength=per_rank)


def reduce_pairs(o: torch.Tensor, pair: torch.Tensor, n_pairs: int) -> torch.Tensor:
    """Sum the rows of o [A, w] that share a pair id, in row order.

    pair [A] must be nondecreasing (the assignments of one pair arrive together, in slot order) and
    every id in [0, n_pairs) must occur; the result is [n_pairs, w], row p the slot-order sum of p's
    rows.  The loop runs over the slot position, at most min(K, experts per rank) times."""
    if pair.numel() and (bool((pair[1:] < pair[:-1]).any()) or int(pair[0]) < 0
                         or int(pair[-1]) >= n_pairs):
        raise ValueError("pair ids must be nondecreasing and inside [0, n_pairs)")
    n = torch.bincount(pair, minlength=n_pairs) if pair.numel() else torch.zeros(n_pairs, dtype=torch.int64, device=pair.device)
    if n_pairs and int(n.min()) == 0:
        raise ValueError("a dispatched pair carries no assignment")
    start = _exclusive_cumsum(n)
    out = torch.zeros((n_pairs,) + tuple(o.shape[1:]), dtype=o.dtype, device=o.device)
    for j in range(int(n.max()) if n_pairs else 0):
        sel = torch.nonzero(n > j).reshape(-1)
        out[sel] += o[start[sel] + j]
    return out


def dispatch_bytes(tokens: int, top_k: int, width: int, elem_bytes: int = 2) -> int:
    """Upper bound on the dispatched row bytes of `tokens` tokens: one row of `width` elements per
    assignment, reached when every expert of a token sits on a different rank (G >= K)."""
    return tokens * top_k * width * elem_bytes


def exchange_bytes(plan: DispatchPlan, width: int, elem_bytes: int = 2, gate_bytes: int = 4) -> dict:
    """Bytes one rank sends in each direction for a plan: latent rows (one per pair) plus the
    assignment metadata (pair index and expert id as int64, the gate) on the way out, one partial
    latent sum per pair (elem_bytes each) on the way back."""
    pairs = int(plan.pair_counts.sum())
    assigns = int(plan.send_counts.sum())
    return {"rows": pairs * width * elem_bytes,
            "metadata": assigns * (2 * 8 + gate_bytes),
            "return": pairs * width * elem_bytes}


def _exchange(send: torch.Tensor, send_counts: list, recv_counts: list, group) -> torch.Tensor:
    out = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    dist.all_to_all_single(out, send.contiguous(), recv_counts, send_counts, group=group)
    return out


def ep_forward(x: torch.Tensor, part: ExpertPartition,
               route: Callable[[torch.Tensor], Tuple[torch.Tensor, torch.Tensor, torch.Tensor]],
               experts: Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor],
               output: Callable[[torch.Tensor, torch.Tensor], torch.Tensor],
               group: Optional["dist.ProcessGroup"] = None, stats: Optional[dict] = None):
    """One expert-parallel forward of this rank's tokens x [T, d].

    route(x)                         -> idx [T, K] (global expert ids), gate [T, K], h [T, l]
    experts(rows, counts, gates)     -> o [R, l]: rows grouped by local expert (counts per local
                                        expert, in order), outputs already multiplied by the gates
    output(z, x)                     -> y [T, d] from the latent sum z [T, l]
    Every rank calls this at the same point (it runs five all-to-alls).  If `stats` is a dict it
    receives this rank's sent pair and assignment counts.  Returns (y, idx, gate)."""
    rank = dist.get_rank(group)
    idx, gate, h = route(x)
    t, k = idx.shape
    width = h.shape[1]
    plan = plan_dispatch(idx, part)
    send_cnt = torch.stack([plan.pair_counts, plan.send_counts], 1).to(torch.int64)   # [G, 2]
    recv_cnt = torch.empty_like(send_cnt)
    dist.all_to_all_single(recv_cnt, send_cnt, group=group)
    pairs_out, assigns_out = plan.pair_counts.tolist(), plan.send_counts.tolist()
    pairs_in, assigns_in = recv_cnt[:, 0].tolist(), recv_cnt[:, 1].tolist()
    if stats is not None:
        stats.update(pairs=int(sum(pairs_out)), assignments=int(sum(assigns_out)))

    # dispatch: one latent row per (token, destination); (pair, expert id) and gate per assignment
    rows = _exchange(h[plan.pair_tok], pairs_out, pairs_in, group)
    meta = torch.stack([plan.assign_pair, idx.reshape(-1)[plan.order].to(torch.int64)], 1)
    meta = _exchange(meta, assigns_out, assigns_in, group)
    gates = _exchange(gate.reshape(-1)[plan.order], assigns_out, assigns_in, group)

    # owner side: pair ids local to each source become ids into `rows`
    src = torch.repeat_interleave(torch.arange(part.world, device=meta.device),
                                  torch.tensor(assigns_in, device=meta.device))
    pin = torch.tensor(pairs_in, dtype=torch.int64, device=meta.device)
    if meta.shape[0] and (bool((meta[:, 0] < 0).any()) or bool((meta[:, 0] >= pin[src]).any())):
        raise ValueError("an assignment names a pair its source did not send")
    pair = _exclusive_cumsum(pin)[src] + meta[:, 0]
    gorder, counts = group_by_local_expert(meta[:, 1], part.first(rank), part.per_rank)
    o_grouped = experts(rows[pair[gorder]], counts, gates[gorder])
    # each pair's slot-order sum, and its trip back, at no less than fp32 (a bf16 sum would add one
    # rounding per pair to z)
    o_arrival = torch.empty(o_grouped.shape, dtype=torch.promote_types(o_grouped.dtype, torch.float32),
                            device=o_grouped.device)
    o_arrival[gorder] = o_grouped.to(o_arrival.dtype)
    partial = reduce_pairs(o_arrival, pair, rows.shape[0])

    # the reverse exchange, then the owner-rank-ordered sum on the source side
    back = _exchange(partial, pairs_in, pairs_out, group)
    z = torch.zeros((t, width), dtype=back.dtype, device=back.device)
    off = 0
    for c in pairs_out:                 # destinations in ascending rank order; tokens distinct in each
        z[plan.pair_tok[off:off + c]] += back[off:off + c]
        off += c
    return output(z, x), idx, gate


def ep_forward_library(layer, x: torch.Tensor, group: Optional["dist.ProcessGroup"] = None,
                       stats: Optional[dict] = None):
    """One expert-parallel forward of this rank's tokens x [T, d] (bf16, on this rank's GPU) with the
    library's three steps on `layer` (a LatentMoE created with ep_world = the group's size and
    ep_rank = this rank).  Every rank calls this at the same point (five all-to-alls).  The plan and
    every row move on the device; the per-destination counts are the one value read on the host.
    Returns (y [T, d] bf16, idx [T, K], gate [T, K])."""
    world = dist.get_world_size(group)
    if layer.ep_world != world:
        raise ValueError("the layer's ep_world must equal the process group's size")
    t, width = x.shape[0], layer.shape.latent
    dev = x.device
    if t:
        plan = layer.ep_dispatch(x)
        send_cnt = plan["counts"].to(torch.int64)
    else:
        plan = None
        send_cnt = torch.zeros((world, 2), dtype=torch.int64, device=dev)
    recv_cnt = torch.empty_like(send_cnt)
    dist.all_to_all_single(recv_cnt, send_cnt, group=group)
    cnt = torch.stack([send_cnt, recv_cnt]).cpu()          # the only host round trip
    pairs_out, assigns_out = cnt[0, :, 0].tolist(), cnt[0, :, 1].tolist()
    pairs_in, assigns_in = cnt[1, :, 0].tolist(), cnt[1, :, 1].tolist()
    if stats is not None:
        stats.update(pairs=int(sum(pairs_out)), assignments=int(sum(assigns_out)))
    p_out, a_out = sum(pairs_out), sum(assigns_out)
    empty = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
    send_rows = plan["send_rows"][:p_out] if plan is not None else empty((0, width), torch.bfloat16)
    send_meta = plan["send_meta"][:a_out] if plan is not None else empty((0, 2), torch.int32)
    send_gate = plan["send_gate"][:a_out] if plan is not None else empty((0,), torch.float32)
    rows = _exchange(send_rows, pairs_out, pairs_in, group)
    meta = _exchange(send_meta, assigns_out, assigns_in, group)
    gates = _exchange(send_gate, assigns_out, assigns_in, group)
    # pair indices local to each source become rows of `rows` (sources arrive in rank order)
    row_base = _exclusive_cumsum(torch.tensor(pairs_in, dtype=torch.int64, device=dev))
    src = torch.repeat_interleave(torch.arange(world, device=dev), torch.tensor(assigns_in, device=dev))
    meta = torch.stack([(meta[:, 0].to(torch.int64) + row_base[src]).to(torch.int32), meta[:, 1]], 1).contiguous()
    partial = layer.ep_experts(rows.contiguous(), meta, gates.contiguous()) if rows.shape[0] else \
        empty((0, width), torch.float32)
    back = _exchange(partial, pairs_in, pairs_out, group)
    if plan is None:
        return empty((0, layer.shape.d), torch.bfloat16), empty((0, layer.shape.top_k), torch.int32), \
            empty((0, layer.shape.top_k), torch.float32)
    y = layer.ep_combine(x, back.contiguous(), plan["tok_pairs"])
    return y, plan["idx"], plan["gate"]
