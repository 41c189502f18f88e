"""The allocation-free routing entry point (lmoe_route_noalloc) against lmoe_forward's routing.

Some callers cannot allocate device memory on their call path (cudaMalloc may synchronise the
device, and a process whose HBM is fully reserved by its own allocator would get an out-of-memory
error).  lmoe_route_noalloc keeps its scratch in the library's static device memory instead.  Here it
is called through the C ABI, twice in a row on the same logits, and each call's outputs must equal
what lmoe_forward produced for the same tokens: expert ids, counts, offsets and grouped rows bit for
bit, gates within the parity tests' gate tolerance.

This file is collected last on purpose; it builds its own layers, so it also passes alone in a fresh
process."""
import ctypes

import numpy as np
import pytest
import torch

import lmoe_inputs as inp
from lmoe_testlib import GATE_TOL, device_weights, host_weights, make_layer, to_dev

pytestmark = pytest.mark.gpu


def _forward_routing(layer, x_np):
    x = to_dev(x_np, "bf16")
    _, idx, gate = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return {"logits": layer.inspect("logits"), "idx": idx, "gate": gate, "counts": layer.inspect("counts"),
            "offsets": layer.inspect("offsets"), "row_of": layer.inspect("row_of")}


def _check_two_calls(ref, t, n, k, bias=None):
    import latentmoe_expert_layer_b200 as lm
    logits = ref["logits"].reshape(t, n).contiguous()
    for _ in range(2):
        idx, gate, counts, offsets, row_of, status = lm.route_noalloc(logits, k, bias)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(idx, ref["idx"])
        assert torch.equal(counts, ref["counts"])
        assert torch.equal(offsets, ref["offsets"])
        assert torch.equal(row_of, ref["row_of"])
        assert float((gate - ref["gate"]).abs().max()) <= GATE_TOL


def test_noalloc_routing_matches_forward_tiny():
    wl = inp.workload("tiny")
    w = inp.make_weights(wl)
    layer = make_layer(wl, w, device_weights(w), wl.tokens)
    ref = _forward_routing(layer, inp.make_x(wl))
    _check_two_calls(ref, wl.tokens, wl.shape.n_experts, wl.shape.top_k)
    layer.close()


def test_noalloc_routing_matches_forward_with_bias():
    wl = inp.workload("tiny")
    w = inp.make_weights(wl)
    w.b_router = np.random.default_rng(5).standard_normal(wl.shape.n_experts).astype(np.float32)
    dev = device_weights(w)
    import latentmoe_expert_layer_b200 as lm
    layer = lm.LatentMoE(wl.shape, wl.tokens, router_bias=True)
    layer.load_weights(dev["w_router"], dev["w_down"], dev["w_up"], dev["w1"], dev["w2"], dev["ws1"], dev["ws2"],
                       b_router=dev["b_router"])
    ref = _forward_routing(layer, inp.make_x(wl))
    _check_two_calls(ref, wl.tokens, wl.shape.n_experts, wl.shape.top_k, bias=dev["b_router"])
    layer.close()


def test_noalloc_routing_matches_forward_decode():
    wl = inp.workload("decode")
    w = host_weights("decode")
    dev = device_weights(w)
    layer = make_layer(wl, w, dev, wl.tokens)
    del dev
    ref = _forward_routing(layer, inp.make_x(wl))
    _check_two_calls(ref, wl.tokens, wl.shape.n_experts, wl.shape.top_k)
    layer.close()
    torch.cuda.empty_cache()


def test_noalloc_rejects_sizes_beyond_its_limit():
    import latentmoe_expert_layer_b200 as lm
    p = ctypes.c_void_p(16)  # never dereferenced: the size checks come first
    s = torch.cuda.current_stream().cuda_stream
    assert lm.lib.lmoe_route_noalloc(p, None, 131072 // 22 + 1, 512, 22, p, p, p, p, p, None, s) == 2
    assert lm.lib.lmoe_route_noalloc(p, None, 16, 2048, 22, p, p, p, p, p, None, s) == 3
    assert lm.lib.lmoe_route_noalloc(p, None, 16, 512, 33, p, p, p, p, p, None, s) == 3
    # a status word that is not 4-byte aligned is rejected before anything is enqueued
    assert lm.lib.lmoe_route_noalloc(p, None, 16, 512, 22, p, p, p, p, p, ctypes.c_void_p(18), s) == 1


def test_noalloc_binding_rejects_wrong_dtypes_and_bias_length():
    """The binding checks dtypes, devices and the bias length before it calls the C ABI, so a bf16
    logits tensor or a short bias raises instead of reaching the kernels."""
    import latentmoe_expert_layer_b200 as lm
    logits = torch.zeros((8, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        lm.route_noalloc(logits.to(torch.bfloat16), 4)
    with pytest.raises(ValueError):
        lm.route_noalloc(logits.cpu(), 4)
    with pytest.raises(ValueError):
        lm.route_noalloc(logits, 4, bias=torch.zeros(63, dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        lm.route_noalloc(logits, 4, bias=torch.zeros(64, dtype=torch.float64, device="cuda"))


@pytest.mark.parametrize("t,n,k", [(300, 64, 8), (256, 512, 22), (129, 32, 32), (77, 48, 1)])
def test_noalloc_exact_ties_match_the_oracle(t, n, k):
    """Integer-valued logits and bias (sums exact in fp32 and fp64) with many exactly equal values:
    the expert ids must follow the tie rule (larger value first, lower expert index among equal
    values) bit for bit, and counts, offsets and grouped rows must equal the oracle's stable grouping
    of the same routing.  Gates agree with the oracle's softmax within the gate tolerance."""
    import latentmoe_expert_layer_b200 as lm
    from oracle import lmoe_oracle as lo
    rng = np.random.default_rng(1000 + t + n + k)
    lg = rng.integers(-3, 4, size=(t, n)).astype(np.float32)
    b = rng.integers(-1, 2, size=n).astype(np.float32)
    ref_logits = lg.astype(np.float64) + b.astype(np.float64)[None, :]
    ref_idx = lo.topk(ref_logits, k)
    ref_gate = lo.softmax_gates(ref_logits, ref_idx)
    counts, offsets, row_of, _ = lo.dispatch(ref_idx, n)
    dl, db = torch.from_numpy(lg).cuda(), torch.from_numpy(b).cuda()
    for _ in range(2):
        idx, gate, c, o, r, status = lm.route_noalloc(dl, k, db)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert np.array_equal(idx.cpu().numpy(), ref_idx)
        assert np.array_equal(c.cpu().numpy(), counts)
        assert np.array_equal(o.cpu().numpy(), offsets)
        assert np.array_equal(r.cpu().numpy(), row_of.reshape(-1))
        assert np.abs(gate.cpu().numpy() - ref_gate).max() <= GATE_TOL
