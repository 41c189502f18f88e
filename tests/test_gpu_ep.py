"""Expert parallelism through the library's three expert-parallel steps (lmoe_ep_dispatch,
lmoe_ep_experts, lmoe_ep_combine), with G ranks simulated in one process on one GPU.

Each rank is its own layer handle holding only its N / G experts.  The two exchanges between the
steps (rows, assignments and gates to their owners; partial sums back to their sources), which
NCCL all-to-alls do across GPUs, are done here by slicing and concatenating device tensors in the
same order.  The assembled y of every rank's tokens must match the oracle's single layer (routing
bit-exact away from near-ties, y within 2e-2 x RMS), and each rank must send exactly one latent row
per distinct (token, owner) pair and one assignment per (token, slot)."""
import dataclasses

import numpy as np
import pytest
import torch

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo
from lmoe_testlib import bf16_to_np, check_routing, check_y, oracle_forward, oracle_routing, to_dev

pytestmark = pytest.mark.gpu

SMALL = inp.LayerShape(d=512, latent=256, n_experts=16, top_k=4, expert_ffn=384, shared_ffn=512)
SUPER128 = dataclasses.replace(inp.SUPER, n_experts=128)


def _layers(shape, w, world, max_tokens):
    import latentmoe_expert_layer_b200 as lm
    nl = shape.n_experts // world
    dev = {k: to_dev(getattr(w, k), "bf16") for k in ("w_router", "w_down", "w_up", "ws1", "ws2")}
    layers = []
    for r in range(world):
        layer = lm.LatentMoE(shape, max_tokens, ep_world=world, ep_rank=r)
        layer.load_weights(dev["w_router"], dev["w_down"], dev["w_up"], to_dev(w.w1[r * nl:(r + 1) * nl], "bf16"),
                           to_dev(w.w2[r * nl:(r + 1) * nl], "bf16"), dev["ws1"], dev["ws2"])
        layers.append(layer)
    torch.cuda.synchronize()
    return layers


def _ep_forward(layers, xs):
    """One forward of every rank's tokens xs[r] through the three steps and emulated exchanges."""
    world = len(layers)
    plans = [layers[r].ep_dispatch(xs[r]) if xs[r].shape[0] else None for r in range(world)]
    counts = [p["counts"].cpu().numpy() if p is not None else np.zeros((world, 2), np.int64) for p in plans]
    pair_off = [np.concatenate([[0], np.cumsum(c[:, 0])]) for c in counts]
    asg_off = [np.concatenate([[0], np.cumsum(c[:, 1])]) for c in counts]
    partials = []
    src_row_off = []   # [owner g][source r]: first row of r's pairs among g's received rows
    for g in range(world):
        rows, meta, gates, off, roff = [], [], [], 0, []
        for r in range(world):
            roff.append(off)
            if plans[r] is None:
                continue
            np_, na = int(counts[r][g, 0]), int(counts[r][g, 1])
            rows.append(plans[r]["send_rows"][pair_off[r][g]:pair_off[r][g] + np_])
            m = plans[r]["send_meta"][asg_off[r][g]:asg_off[r][g] + na].clone()
            m[:, 0] += off
            meta.append(m)
            gates.append(plans[r]["send_gate"][asg_off[r][g]:asg_off[r][g] + na])
            off += np_
        src_row_off.append(roff)
        rows = torch.cat(rows) if rows else torch.empty((0, layers[g].shape.latent), dtype=torch.bfloat16,
                                                        device="cuda")
        meta = torch.cat(meta) if meta else torch.empty((0, 2), dtype=torch.int32, device="cuda")
        gates = torch.cat(gates) if gates else torch.empty((0,), dtype=torch.float32, device="cuda")
        partials.append(layers[g].ep_experts(rows, meta.contiguous(), gates.contiguous()) if rows.shape[0]
                        else torch.empty((0, layers[g].shape.latent), dtype=torch.float32, device="cuda"))
    ys = []
    for r in range(world):
        if plans[r] is None:
            ys.append(torch.empty((0, layers[r].shape.d), dtype=torch.bfloat16, device="cuda"))
            continue
        back = torch.cat([partials[g][src_row_off[g][r]:src_row_off[g][r] + int(counts[r][g, 0])]
                          for g in range(world)])
        ys.append(layers[r].ep_combine(xs[r], back.contiguous(), plans[r]["tok_pairs"]))
    torch.cuda.synchronize()
    for layer in layers:
        assert layer.device_status() == 0
    return ys, plans, counts


@pytest.mark.parametrize("shape,world,tokens", [(SMALL, 2, [40, 23]), (SMALL, 4, [17, 0, 33, 5]),
                                                 (SUPER128, 4, [16, 11, 24, 13])],
                         ids=["small-G2", "small-G4-empty-rank", "super128-G4"])
def test_ep_steps_assemble_the_single_gpu_layer(shape, world, tokens):
    wl = inp.Workload("ep", shape, sum(tokens), 7, 8, "bf16", "bf16")
    w = inp.make_weights(wl)
    x_all = inp.make_x(wl)
    starts = np.concatenate([[0], np.cumsum(tokens)])
    xs = [to_dev(x_all[starts[r]:starts[r + 1]], "bf16") for r in range(world)]
    layers = _layers(shape, w, world, max(tokens))
    try:
        ys, plans, counts = _ep_forward(layers, xs)
        ow = lo.OracleWeights(w)
        x64 = lo.lift(x_all, "bf16")
        full = oracle_routing(ow, x64, shape.top_k)
        nl = shape.n_experts // world
        idx_all = np.concatenate([p["idx"].cpu().numpy() for p in plans if p is not None])
        gate_all = np.concatenate([p["gate"].cpu().numpy() for p in plans if p is not None])
        diff, _ = check_routing(idx_all, gate_all, full, shape.top_k)
        ref = oracle_forward(ow, x64, shape.top_k)
        yref = ref["y"].copy()
        if diff.any():
            yref[diff] = oracle_forward(ow, x64[diff], shape.top_k, idx=idx_all[diff])["y"]
        y_all = np.concatenate([bf16_to_np(y) for y in ys])
        rel = check_y(y_all, yref)
        # one latent row per distinct (token, owner) pair, one assignment per (token, slot)
        for r in range(world):
            if plans[r] is None:
                continue
            idx_r = plans[r]["idx"].cpu().numpy()
            owners = idx_r // nl
            for g in range(world):
                assert counts[r][g, 0] == int((owners == g).any(axis=1).sum())
                assert counts[r][g, 1] == int((owners == g).sum())
        print(f"EP {shape.n_experts} experts over {world} ranks: max|err|/RMS {rel:.3g}")
    finally:
        for layer in layers:
            layer.close()
        torch.cuda.empty_cache()


def test_ep_layer_rejects_the_single_gpu_forward():
    import latentmoe_expert_layer_b200 as lm
    layer = lm.LatentMoE(SMALL, 8, ep_world=2, ep_rank=1)
    x = torch.zeros((4, SMALL.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lm.LmoeError) as e:
        layer.forward(x)
    assert e.value.code == 6 or e.value.code == 3   # not loaded, or unsupported once loaded
    layer.close()


class _ThreadRanks:
    """Stand-in for the two torch.distributed calls ep_forward_library makes (get_world_size and
    all_to_all_single), for ranks that are host threads of one process: each rank deposits its input
    chunks, and after a barrier takes the chunks addressed to it, in source-rank order.  Only the
    host threads meet here; no kernel waits on another rank's kernel."""

    def __init__(self, world):
        import threading
        self.world = world
        self.barrier = threading.Barrier(world, timeout=120)
        self.slots = [None] * world
        self.rank_of = {}

    def get_world_size(self, group=None):
        return self.world

    def all_to_all_single(self, out, inp, output_split_sizes=None, input_split_sizes=None, group=None):
        import threading
        r = self.rank_of[threading.get_ident()]
        sizes = input_split_sizes or [inp.shape[0] // self.world] * self.world
        offs = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
        self.slots[r] = [inp[offs[g]:offs[g + 1]] for g in range(self.world)]
        self.barrier.wait()
        parts = [self.slots[src][r] for src in range(self.world)]
        if out.numel():
            out.copy_(torch.cat(parts))
        self.barrier.wait()


@pytest.mark.parametrize("world,tokens", [(2, [21, 30]), (4, [9, 14, 0, 25])])
def test_ep_forward_library_over_thread_ranks(world, tokens, monkeypatch):
    """ep.ep_forward_library end to end (plan, the five all-to-alls, the three library steps),
    with the collectives replaced by _ThreadRanks; y of every rank matches the oracle's layer."""
    import threading

    from latentmoe_expert_layer_b200 import ep
    wl = inp.Workload("ep", SMALL, sum(tokens), 9, 10, "bf16", "bf16")
    w = inp.make_weights(wl)
    x_all = inp.make_x(wl)
    starts = np.concatenate([[0], np.cumsum(tokens)])
    xs = [to_dev(x_all[starts[r]:starts[r + 1]], "bf16") for r in range(world)]
    layers = _layers(SMALL, w, world, max(tokens))
    fake = _ThreadRanks(world)
    monkeypatch.setattr(ep, "dist", fake)
    out, errors = [None] * world, []

    def run(r):
        try:
            fake.rank_of[threading.get_ident()] = r
            stats = {}
            y, idx, gate = ep.ep_forward_library(layers[r], xs[r], stats=stats)
            torch.cuda.synchronize()
            out[r] = (bf16_to_np(y), idx.cpu().numpy(), gate.cpu().numpy(), stats)
        except Exception as e:  # pragma: no cover - reported below
            errors.append(e)
            fake.barrier.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    try:
        for th in threads:
            th.start()
        for th in threads:
            th.join(timeout=300)
        assert not errors, errors
        for layer in layers:
            assert layer.device_status() == 0
        ow = lo.OracleWeights(w)
        x64 = lo.lift(x_all, "bf16")
        full = oracle_routing(ow, x64, SMALL.top_k)
        idx_all = np.concatenate([o[1] for o in out])
        gate_all = np.concatenate([o[2] for o in out])
        diff, _ = check_routing(idx_all, gate_all, full, SMALL.top_k)
        ref = oracle_forward(ow, x64, SMALL.top_k)
        yref = ref["y"].copy()
        if diff.any():
            yref[diff] = oracle_forward(ow, x64[diff], SMALL.top_k, idx=idx_all[diff])["y"]
        rel = check_y(np.concatenate([o[0] for o in out]), yref)
        for r in range(world):
            assert out[r][3]["assignments"] == tokens[r] * SMALL.top_k
        print(f"ep_forward_library over {world} thread ranks: max|err|/RMS {rel:.3g}")
    finally:
        for layer in layers:
            layer.close()
