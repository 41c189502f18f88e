"""Parity of the CUDA layer (through the C ABI) against the fp64 oracle on seeded inputs.

Routing must match bit for bit except on logit near-ties (gap < 1e-5), the dispatch maps must be
exactly the grouping the oracle derives from the GPU's own routing, and y must be within
2e-2 x RMS(y) of the oracle (tokens whose routing differs at a near-tie are re-evaluated by the
oracle with the GPU's routing)."""
import dataclasses

import numpy as np
import pytest
import torch

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo
from lmoe_testlib import (Y_TOL_BF16, bf16_to_np, check_dispatch, compare_bf16, device_weights, host_weights,
                          make_layer, oracle_weights, run_layer, to_dev)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------------------------ tiny
@pytest.fixture(scope="module")
def tiny():
    wl = inp.workload("tiny")
    w = inp.make_weights(wl)
    dev = device_weights(w)
    layer = make_layer(wl, w, dev, wl.tokens)
    yield wl, w, layer
    layer.close()


def test_tiny_full_parity(tiny):
    wl, w, layer = tiny
    x = inp.make_x(wl)
    st = compare_bf16(layer, oracle_weights(w, False), x, wl.shape.top_k)
    check_dispatch(layer, st["idx"], wl.shape.n_experts)


def test_tiny_latent_h(tiny):
    wl, w, layer = tiny
    x = inp.make_x(wl)
    run_layer(layer, x)
    h = bf16_to_np(layer.inspect("h").view(torch.bfloat16)).reshape(wl.tokens, wl.shape.latent)
    ow = oracle_weights(w, False)
    href = lo.lift(x, "bf16") @ ow.w_down.T
    assert np.abs(h - href).max() <= 2 ** -7 * np.abs(href).max()


@pytest.mark.parametrize("t", [1, 2, 7, 33, 63])
def test_tiny_ragged_tokens(tiny, t):
    wl, w, layer = tiny
    x = inp.make_x(wl, tokens=t)
    compare_bf16(layer, oracle_weights(w, False), x, wl.shape.top_k)


@pytest.mark.parametrize("t", [600, 1000])
def test_tiny_shape_at_prefill_sizes(t):
    """Past 512 tokens the dense and grouped GEMMs run as CTA pairs over 256 weight rows.  The tiny
    layer's weight blocks are narrower than a pair (router 16 rows, W_down 64, experts 128 and 64), so
    the odd CTA of every pair holds no valid rows, and the token tiles end ragged."""
    wl = dataclasses.replace(inp.workload("tiny"), tokens=t)
    w = inp.make_weights(wl)
    layer = make_layer(wl, w, device_weights(w), t)
    try:
        st = compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl), wl.shape.top_k)
        check_dispatch(layer, st["idx"], wl.shape.n_experts)
    finally:
        layer.close()


def test_tiny_deterministic(tiny):
    wl, w, layer = tiny
    x = inp.make_x(wl)
    a = run_layer(layer, x)
    b = run_layer(layer, x)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_zero_tokens_and_too_many(tiny):
    import latentmoe_expert_layer_b200 as lm
    wl, w, layer = tiny
    x = torch.empty((0, wl.shape.d), dtype=torch.bfloat16, device="cuda")
    y, idx, gate = layer.forward(x)
    assert y.shape == (0, wl.shape.d)
    xb = to_dev(inp.make_x(wl), "bf16")
    big = torch.cat([xb, xb])
    with pytest.raises(lm.LmoeError) as e:
        layer.forward(big)
    assert e.value.code == 2


# ------------------------------------------------------------------------------------------------ Super
@pytest.fixture(scope="module")
def superlayer():
    wl = inp.workload("decode")
    w = host_weights("decode")
    dev = device_weights(w)
    layer = make_layer(wl, w, dev, inp.workload("prefill").tokens)
    yield w, dev, layer
    layer.close()
    del dev
    torch.cuda.empty_cache()


def test_decode_full_parity(superlayer):
    w, _, layer = superlayer
    wl = inp.workload("decode")
    st = compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl), wl.shape.top_k)
    check_dispatch(layer, st["idx"], wl.shape.n_experts)
    print(f"decode: rel err {st['rel_err']:.3g}, logit err {st['logit_err']:.3g}, near ties {st['near_ties']}, "
          f"routing diffs {st['routing_diffs']}")


@pytest.mark.parametrize("t", [1, 5, 100, 257, 513])
def test_super_ragged_tokens(superlayer, t):
    w, _, layer = superlayer
    wl = inp.workload("prefill")
    x = inp.make_x(wl, tokens=t)
    compare_bf16(layer, oracle_weights(w, False), x, wl.shape.top_k)


def test_prefill_sampled_parity_and_full_dispatch(superlayer):
    w, _, layer = superlayer
    wl = inp.workload("prefill")
    x = inp.make_x(wl)
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, 1, wl.tokens - 1], rng.choice(wl.tokens, 40, replace=False)]))
    st = compare_bf16(layer, oracle_weights(w, False), x, wl.shape.top_k, tokens=sample)
    check_dispatch(layer, st["idx"], wl.shape.n_experts)
    print(f"prefill: rel err {st['rel_err']:.3g} on {st['tokens_y_checked']} tokens, logit err "
          f"{st['logit_err']:.3g}, routing checked on {st['tokens_routed_checked']} tokens, near ties "
          f"{st['near_ties']}, routing diffs {st['routing_diffs']}")


def test_decode_host_forward_matches_device_forward(superlayer):
    """lmoe_forward_host at decode size (one call, no chunks): copies in, the layer, copies out, all on
    the caller's stream; the results equal the device-buffer forward's bit for bit, and a call with
    NULL idx / gate outputs still writes y."""
    _, _, layer = superlayer
    wl = inp.workload("decode")
    x_np = inp.make_x(wl)
    y_dev, idx_dev, gate_dev = run_layer(layer, x_np)
    xh = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.zeros((wl.tokens, wl.shape.d), dtype=torch.bfloat16).pin_memory()
    ih = torch.empty((wl.tokens, wl.shape.top_k), dtype=torch.int32).pin_memory()
    gh = torch.empty((wl.tokens, wl.shape.top_k), dtype=torch.float32).pin_memory()
    layer.forward_host(xh, yh, ih, gh)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert np.array_equal(bf16_to_np(yh), y_dev)
    assert np.array_equal(ih.numpy(), idx_dev) and np.array_equal(gh.numpy(), gate_dev)
    yh.zero_()
    layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_to_np(yh), y_dev)


def test_prefill_host_forward_in_chunks_matches_device_forward(superlayer):
    """lmoe_forward_host splits the 16384-token batch into 4096-token chunks whose copies overlap the
    neighbouring chunks' compute.  Every token's routing equals the one-call device forward's bit for
    bit; y equals it within the parity tolerance (the chunks' expert-up GEMM runs as CTA pairs, the
    one-call forward's on one CTA)."""
    w, _, layer = superlayer
    wl = inp.workload("prefill")
    x_np = inp.make_x(wl)
    y_dev, idx_dev, gate_dev = run_layer(layer, x_np)
    xh = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty((wl.tokens, wl.shape.d), dtype=torch.bfloat16).pin_memory()
    ih = torch.empty((wl.tokens, wl.shape.top_k), dtype=torch.int32).pin_memory()
    gh = torch.empty((wl.tokens, wl.shape.top_k), dtype=torch.float32).pin_memory()
    for _ in range(2):  # twice: the second call's input copies must wait for the first call's layer
        yh.zero_()
        layer.forward_host(xh, yh, ih, gh)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        assert np.array_equal(ih.numpy(), idx_dev)
        assert np.array_equal(gh.numpy(), gate_dev)
        y_host = bf16_to_np(yh)
        rms = np.sqrt(np.mean(y_dev ** 2))
        err = np.abs(y_host - y_dev).max()
        assert err <= Y_TOL_BF16 * rms, f"chunked host forward differs: {err:.3g} vs RMS {rms:.3g}"
    print(f"prefill host forward in chunks: max|dy|/RMS {err / rms:.3g}, "
          f"bit-identical y: {bool(np.array_equal(y_host, y_dev))}")


@pytest.fixture(scope="module")
def skewlayer(superlayer):
    w, dev, _ = superlayer
    wl = inp.workload("skewed")
    layer = make_layer(wl, w, dev, wl.tokens)
    yield layer
    layer.close()


def test_skewed_sampled_parity(skewlayer, superlayer):
    w, _, _ = superlayer
    layer = skewlayer
    wl = inp.workload("skewed")
    x = inp.make_x(wl)
    rng = np.random.default_rng(1)
    sample = np.unique(np.concatenate([[0, wl.tokens - 1], rng.choice(wl.tokens, 40, replace=False)]))
    st = compare_bf16(layer, oracle_weights(w, True), x, wl.shape.top_k, tokens=sample)
    check_dispatch(layer, st["idx"], wl.shape.n_experts)
    print(f"skewed: rel err {st['rel_err']:.3g} on {st['tokens_y_checked']} tokens, logit err {st['logit_err']:.3g}, "
          f"routing checked on {st['tokens_routed_checked']} tokens, near ties {st['near_ties']}, routing diffs "
          f"{st['routing_diffs']}")
    counts = np.bincount(st["idx"].ravel(), minlength=wl.shape.n_experts)
    assert (counts == 0).sum() >= 32 and counts.max() > 0.1 * wl.tokens


def test_wait_timeout_reported_and_context_survives(tiny):
    """Failure detection without a fault: a kernel waits, bounded, on a barrier nothing arrives on.
    The timeout reaches the host as LMOE_ERR_DEVICE_TIMEOUT, the status word is cleared by reading
    it, and the context still runs the layer with unchanged results."""
    wl, w, layer = tiny
    x = inp.make_x(wl)
    before = run_layer(layer, x)
    layer.selftest_wait_timeout(2_000_000)  # 2 ms
    torch.cuda.synchronize()
    assert layer.device_status() == 7
    assert layer.device_status() == 0
    after = run_layer(layer, x)
    for a, b in zip(before, after):
        assert np.array_equal(a, b)


# ------------------------------------------------------------------------------------------------ standard MoE
@pytest.fixture(scope="module")
def stdlayer():
    """The standard MoE of the Super budget (latent = 0: N = 128, K = 6, experts d -> m -> d)."""
    wl = inp.workload("standard_decode")
    w = inp.make_weights(wl)
    layer = make_layer(wl, w, device_weights(w), inp.workload("standard_prefill").tokens)
    torch.cuda.empty_cache()
    yield w, layer
    layer.close()
    torch.cuda.empty_cache()


def test_standard_decode_parity_and_dispatch(stdlayer):
    w, layer = stdlayer
    wl = inp.workload("standard_decode")
    st = compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl), wl.shape.top_k)
    check_dispatch(layer, st["idx"], wl.shape.n_experts)
    print(f"standard decode: rel err {st['rel_err']:.3g}, logit err {st['logit_err']:.3g}")


@pytest.mark.parametrize("t", [3, 600])
def test_standard_ragged_tokens(stdlayer, t):
    w, layer = stdlayer
    wl = inp.workload("standard_prefill")
    compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl, tokens=t), wl.shape.top_k,
             tokens=np.unique([0, t // 2, t - 1]))


def test_standard_prefill_sampled_parity(stdlayer):
    w, layer = stdlayer
    wl = inp.workload("standard_prefill")
    st = compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl), wl.shape.top_k, tokens=[0, 8191, wl.tokens - 1])
    check_dispatch(layer, st["idx"], wl.shape.n_experts)


def test_standard_rejects_projections_and_nvfp4():
    import latentmoe_expert_layer_b200 as lm
    with pytest.raises(RuntimeError):
        lm.LatentMoE(inp.STANDARD, 16, precision="nvfp4")
    w = inp.make_weights(inp.workload("tiny"))
    layer = lm.LatentMoE(dataclasses.replace(inp.TINY, latent=0), 16)
    dev = device_weights(w)
    with pytest.raises(RuntimeError):     # W_down / W_up given to a layer without projections
        layer.load_weights(dev["w_router"], dev["w_down"], dev["w_up"], dev["w1"], dev["w2"], dev["ws1"], dev["ws2"])
    layer.close()


def test_cuda_graph_replay_matches_eager(superlayer):
    """lmoe_forward makes no host synchronisation or allocation, so a forward can be captured in a
    CUDA graph; replaying it gives the eager call's outputs bit for bit."""
    _, _, layer = superlayer
    wl = inp.workload("decode")
    x = to_dev(inp.make_x(wl), "bf16")
    y = torch.empty((wl.tokens, wl.shape.d), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((wl.tokens, wl.shape.top_k), dtype=torch.int32, device="cuda")
    gate = torch.empty((wl.tokens, wl.shape.top_k), dtype=torch.float32, device="cuda")
    layer.forward(x, y, idx, gate)
    torch.cuda.synchronize()
    ref = (y.clone(), idx.clone(), gate.clone())
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                 # warm-up on the stream the capture will use
        layer.forward(x, y, idx, gate)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.forward(x, y, idx, gate)
    for t in (y, idx, gate):
        t.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(y, ref[0]) and torch.equal(idx, ref[1]) and torch.equal(gate, ref[2])
    del graph


@pytest.mark.parametrize("k", [1, 16])
def test_degenerate_top_k(k):
    """K = 1 (every gate exactly 1) and K = N (every expert selected, softmax over all logits), on
    the tiny layer's weights."""
    base = inp.workload("tiny")
    wl = dataclasses.replace(base, shape=dataclasses.replace(base.shape, top_k=k))
    w = inp.make_weights(base)
    layer = make_layer(wl, w, device_weights(w), wl.tokens)
    try:
        st = compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl), k)
        check_dispatch(layer, st["idx"], wl.shape.n_experts)
        if k == 1:
            assert np.all(st["gate"] == 1.0)
        else:
            assert np.array_equal(np.sort(st["idx"], axis=1), np.tile(np.arange(16), (wl.tokens, 1)))
    finally:
        layer.close()


def test_a_second_layer_does_not_disturb_the_first(superlayer):
    """Kernel attributes are process-wide: creating a layer of another shape (here N = 16 experts)
    must not change what an existing layer's forward can launch."""
    import latentmoe_expert_layer_b200 as lm
    w, _, layer = superlayer
    wl = inp.workload("decode")
    small = lm.LatentMoE(dataclasses.replace(inp.TINY, latent=0), 16)
    try:
        compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl, tokens=64), wl.shape.top_k)
    finally:
        small.close()
