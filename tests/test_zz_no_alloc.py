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
        idx, gate, counts, offsets, row_of = lm.route_noalloc(logits, k, bias)
        torch.cuda.synchronize()
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
    assert lm.lib.lmoe_route_noalloc(p, None, 131072 // 22 + 1, 512, 22, p, p, p, p, p, s) == 2
    assert lm.lib.lmoe_route_noalloc(p, None, 16, 2048, 22, p, p, p, p, p, s) == 3
    assert lm.lib.lmoe_route_noalloc(p, None, 16, 512, 33, p, p, p, p, p, s) == 3
