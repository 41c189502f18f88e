"""Expert-parallel data movement (latentmoe_expert_layer_b200.ep) on CPU ranks over gloo.

The compute steps are the oracle's (test side only); the module under test moves the latent rows
(one per (token, destination rank) pair), the assignments' expert ids and gates, and the pre-reduced
partial sums between ranks.  Every rank's y must equal the single-process oracle layer on its tokens,
for several world sizes, ragged token counts and a rank without tokens."""
import math
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from latentmoe_expert_layer_b200 import ep  # noqa: E402
from oracle import lmoe_oracle as lo  # noqa: E402

D, L, N, K, M, MS = 8, 4, 16, 3, 6, 5


class _W:
    """A small float64 layer (router, W_down, W_up, experts, shared expert)."""

    def __init__(self, seed):
        rng = np.random.default_rng(seed)
        self.w_router = rng.standard_normal((N, D))
        self.b_router = None
        self.w_down = rng.standard_normal((L, D)) / math.sqrt(D)
        self.w_up = rng.standard_normal((D, L)) / math.sqrt(L)
        self._w1 = rng.standard_normal((N, M, L)) / math.sqrt(L)
        self._w2 = rng.standard_normal((N, L, M)) / math.sqrt(M)
        self.ws1 = rng.standard_normal((MS, D)) / math.sqrt(D)
        self.ws2 = rng.standard_normal((D, MS)) / math.sqrt(MS)
        self.n_experts = N

    def w1(self, e):
        return self._w1[e]

    def w2(self, e):
        return self._w2[e]


def _tokens(world):
    counts = [5 + 3 * r for r in range(world)]
    if world >= 4:
        counts[2] = 0            # a rank without tokens still takes part in every exchange
    return counts


def _callables(W, rank, part):
    def route(x):
        xn = x.numpy()
        logits = lo.router_logits(xn, W.w_router)
        idx = lo.topk(logits, K)
        gate = lo.softmax_gates(logits, idx)
        return torch.from_numpy(idx), torch.from_numpy(gate), torch.from_numpy(xn @ W.w_down.T)

    def experts(rows, counts, gates):
        out = torch.empty_like(rows)
        off = 0
        for e_local, c in enumerate(counts.tolist()):
            e = part.first(rank) + e_local
            r = rows[off:off + c].numpy()
            o = lo.sqrelu(r @ W.w1(e).T) @ W.w2(e).T
            out[off:off + c] = torch.from_numpy(o) * gates[off:off + c, None]
            off += c
        return out

    def output(z, x):
        s = lo.sqrelu(x.numpy() @ W.ws1.T) @ W.ws2.T
        return torch.from_numpy(z.numpy() @ W.w_up.T + s)

    return route, experts, output


def _bf16_callables(W, rank, part):
    """The oracle's steps with bf16 latent rows and bf16 expert outputs, as a bf16 device layer would
    send and produce them."""
    route, experts, output = _callables(W, rank, part)

    def route16(x):
        idx, gate, h = route(x)
        return idx, gate, h.to(torch.bfloat16)

    def experts16(rows, counts, gates):
        return experts(rows.to(torch.float64), counts, gates.to(torch.float64)).to(torch.bfloat16)

    def output16(z, x):
        return output(z.to(torch.float64), x)

    return route16, experts16, output16


def _worker_bf16(rank, world, init_file, q):
    import datetime
    dist.init_process_group("gloo", init_method="file://" + init_file, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        W = _W(5)
        counts = _tokens(world)
        x_all = np.random.default_rng(6).standard_normal((sum(counts), D))
        start = sum(counts[:rank])
        x = torch.from_numpy(x_all[start:start + counts[rank]].copy())
        part = ep.ExpertPartition(N, world)
        y, idx, _ = ep.ep_forward(x, part, *_bf16_callables(W, rank, part))
        ref = lo.forward(W, x_all, K)
        sl = slice(start, start + counts[rank])
        rms = float(np.sqrt(np.mean(ref["y"] ** 2)))
        err = float(np.abs(y.numpy() - ref["y"][sl]).max()) if counts[rank] else 0.0
        q.put((rank, err / rms, bool(np.array_equal(idx.numpy(), ref["idx"][sl]))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ep_forward_with_bf16_rows_stays_within_the_bf16_tolerance(world, tmp_path):
    """bf16 rows and bf16 expert outputs: the pair partial sums travel at fp32, so y stays within
    the layer's bf16 tolerance (2e-2 x RMS) of the fp64 oracle."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    init_file = str(tmp_path / "rendezvous")
    procs = [ctx.Process(target=_worker_bf16, args=(r, world, init_file, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, rel, same_idx in res:
        assert same_idx
        assert rel < 2e-2, (rank, rel)


def _worker(rank, world, init_file, q):
    import datetime
    # rendezvous through a file in the test's own temporary directory (no port to race for)
    dist.init_process_group("gloo", init_method="file://" + init_file, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        W = _W(5)
        counts = _tokens(world)
        x_all = np.random.default_rng(6).standard_normal((sum(counts), D))
        start = sum(counts[:rank])
        x = torch.from_numpy(x_all[start:start + counts[rank]].copy())
        part = ep.ExpertPartition(N, world)
        stats = {}
        y, idx, gate = ep.ep_forward(x, part, *_callables(W, rank, part), stats=stats)
        ref = lo.forward(W, x_all, K)
        sl = slice(start, start + counts[rank])
        owners = {(t, int(e) // part.per_rank) for t, row in enumerate(ref["idx"][sl]) for e in row}
        q.put((rank, np.abs(y.numpy() - ref["y"][sl]).max() if counts[rank] else 0.0,
               bool(np.array_equal(idx.numpy(), ref["idx"][sl])), y.shape[0],
               stats["pairs"] == len(owners), stats["assignments"] == counts[rank] * K))
    finally:
        dist.destroy_process_group()



@pytest.mark.parametrize("world", [2, 4])
def test_ep_forward_matches_single_process_layer(world, tmp_path):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    init_file = str(tmp_path / "rendezvous")
    procs = [ctx.Process(target=_worker, args=(r, world, init_file, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    counts = _tokens(world)
    for rank, err, same_idx, n, pairs_ok, assigns_ok in res:
        assert n == counts[rank]
        assert same_idx
        assert pairs_ok and assigns_ok      # one latent row per distinct (token, owner) pair
        assert err < 1e-12, (rank, err)


def test_dispatch_plan_groups_by_owner_in_token_slot_order():
    rng = np.random.default_rng(7)
    idx = torch.from_numpy(np.stack([rng.choice(N, K, replace=False) for _ in range(11)]))
    part = ep.ExpertPartition(N, 4)
    plan = ep.plan_dispatch(idx, part)
    order = plan.order.numpy()
    assert sorted(order.tolist()) == list(range(idx.numel()))          # every assignment once
    owners = (idx.reshape(-1).numpy() // part.per_rank)[order]
    assert np.all(np.diff(owners) >= 0)                                  # grouped by destination
    for r in range(4):
        a = order[owners == r]
        assert np.all(np.diff(a) > 0)                                    # (token, slot) order inside
        assert len(a) == plan.send_counts[r]


def test_grouping_by_local_expert_is_stable_and_checks_ownership():
    eids = torch.tensor([9, 8, 9, 11, 8, 8])
    order, counts = ep.group_by_local_expert(eids, first=8, per_rank=4)
    assert order.tolist() == [1, 4, 5, 0, 2, 3] and counts.tolist() == [3, 2, 0, 1]
    with pytest.raises(ValueError):
        ep.group_by_local_expert(torch.tensor([3]), first=8, per_rank=4)
    with pytest.raises(ValueError):
        ep.ExpertPartition(10, 4)


def test_latent_dispatch_moves_d_over_l_fewer_bytes():
    # Super shape: d = 4096, l = 1024, K = 22; the latent rows are 4x smaller than rows in d
    assert ep.dispatch_bytes(256, 22, 1024) * 4 == ep.dispatch_bytes(256, 22, 4096)
    assert ep.dispatch_bytes(1, 22, 1024) == 22 * 1024 * 2


def _pairs_bruteforce(idx, part):
    """(token, owner) pairs sorted by (owner, token), and each assignment's pair index within its
    owner's segment, by plain loops."""
    pairs = sorted({(int(e) // part.per_rank, t) for t, row in enumerate(idx.tolist()) for e in row})
    seg = {}
    for o, t in pairs:
        seg.setdefault(o, []).append(t)
    sent = sorted(((int(e) // part.per_rank, t, s) for t, row in enumerate(idx.tolist())
                   for s, e in enumerate(row)))
    return pairs, [seg[o].index(t) for o, t, _ in sent]


@pytest.mark.parametrize("world", [1, 2, 4, 8, 16])
def test_pairs_match_bruteforce(world):
    rng = np.random.default_rng(11 + world)
    idx = torch.from_numpy(np.stack([rng.choice(N, K, replace=False) for _ in range(13)]))
    part = ep.ExpertPartition(N, world)
    plan = ep.plan_dispatch(idx, part)
    pairs, assign_pair = _pairs_bruteforce(idx, part)
    assert plan.pair_tok.tolist() == [t for _, t in pairs]
    assert plan.pair_counts.tolist() == [sum(1 for o, _ in pairs if o == r) for r in range(world)]
    assert plan.assign_pair.tolist() == assign_pair
    assert int(plan.pair_counts.sum()) <= min(K, world) * idx.shape[0]
    if world == 1:                                           # one rank: every token is one pair
        assert plan.pair_tok.tolist() == list(range(idx.shape[0]))
    if world == N:                                           # one expert per rank: a pair per assignment
        assert int(plan.pair_counts.sum()) == idx.numel()


def test_plan_of_no_tokens_is_empty():
    plan = ep.plan_dispatch(torch.zeros((0, K), dtype=torch.int64), ep.ExpertPartition(N, 4))
    assert plan.pair_tok.numel() == 0 and plan.order.numel() == 0
    assert plan.pair_counts.tolist() == [0] * 4 and plan.send_counts.tolist() == [0] * 4


def test_reduce_pairs_sums_in_row_order_and_checks_ids():
    o = torch.tensor([[1.0], [2.0], [4.0], [8.0], [16.0]], dtype=torch.float64)
    out = ep.reduce_pairs(o, torch.tensor([0, 0, 1, 2, 2]), 3)
    assert out.reshape(-1).tolist() == [3.0, 4.0, 24.0]
    # the order is the row order: (1e16 + 1) - 1e16 loses the 1, 1e16 - 1e16 + 1 keeps it
    big = torch.tensor([[1e16], [1.0], [-1e16]], dtype=torch.float64)
    assert float(ep.reduce_pairs(big, torch.tensor([0, 0, 0]), 1)) == 0.0
    assert float(ep.reduce_pairs(big[[0, 2, 1]], torch.tensor([0, 0, 0]), 1)) == 1.0
    assert ep.reduce_pairs(o[:0], torch.zeros(0, dtype=torch.int64), 0).shape == (0, 1)
    for bad, n in (([1, 0, 0, 1, 2], 3), ([0, 0, 1, 2, 3], 3), ([0, 0, 2, 2, 2], 3)):
        with pytest.raises(ValueError):
            ep.reduce_pairs(o, torch.tensor(bad), n)


def test_exchange_bytes_at_the_super_shape():
    # Super shape (l = 1024, N = 512, K = 22) over 8 ranks: at most 8 latent rows per token leave a
    # rank instead of 22, and the same count of partial sums comes back
    rng = np.random.default_rng(3)
    t = 64
    idx = torch.from_numpy(np.stack([rng.choice(512, 22, replace=False) for _ in range(t)]))
    plan = ep.plan_dispatch(idx, ep.ExpertPartition(512, 8))
    b = ep.exchange_bytes(plan, 1024)
    pairs = int(plan.pair_counts.sum())
    assert b["rows"] == b["return"] == pairs * 1024 * 2
    assert b["metadata"] == t * 22 * 20
    assert b["rows"] <= 8 * t * 1024 * 2 < ep.dispatch_bytes(t, 22, 1024)
