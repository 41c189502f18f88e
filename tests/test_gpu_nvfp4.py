"""NVFP4 path (routed and shared experts in E2M1 with E4M3 16-element block scales and an fp32 tensor
scale) against the oracle's own NVFP4 quantiser and forward.

Weights: the library quantises on the device; the codes, block scales and tensor scales it exports
must equal the oracle's bytes exactly (both decide in fp32 with the same rules).  Layer output: within
5e-2 x RMS(y) of the oracle's NVFP4 forward (router, W_down and W_up at the device's bf16 values)."""
import numpy as np
import pytest
import torch

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo
from oracle import nvfp4 as nv
from lmoe_testlib import (bf16_to_np, check_routing, check_y, device_weights, host_weights, make_layer,
                          oracle_weights, to_dev)

pytestmark = pytest.mark.gpu
Y_TOL_NVFP4 = 5e-2


def _pack(codes):
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def _check_weight_bytes(layer, w, which, index):
    src = {0: lambda: w.w1[index], 1: lambda: w.w2[index], 2: lambda: w.ws1, 3: lambda: w.ws2}[which]()
    ref_c, ref_s, ref_g = nv.quantize(inp.bf16_bits_to_f32(src))
    codes, scales, g = layer.export_nvfp4(which, index)
    assert g == ref_g, (which, index, g, ref_g)
    assert np.array_equal(scales, ref_s), (which, index, np.argwhere(scales != ref_s)[:5])
    assert np.array_equal(codes, _pack(ref_c)), (which, index, np.argwhere(codes != _pack(ref_c))[:5])


def _run(layer, x_np):
    x = to_dev(x_np, "bf16")
    y, idx, gate = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return bf16_to_np(y), idx.cpu().numpy(), gate.cpu().numpy()


def _compare_nvfp4(layer, w, x_np, k, tokens=None):
    y, idx, gate = _run(layer, x_np)
    ow = oracle_weights(w, False)
    x64 = lo.lift(x_np, "bf16")
    # the per-call activation scales come from the whole batch (oracle's own x and bf16 h)
    g_x = nv.tensor_scale(x64.astype(np.float32))
    g_h = nv.tensor_scale(nv.bf16_round(x64 @ ow.w_down.T).astype(np.float32))
    sel = np.arange(x_np.shape[0]) if tokens is None else np.asarray(tokens)
    ref = nv.forward_nvfp4(ow, x64[sel], k, g_x=g_x, g_h=g_h)
    diff, near = check_routing(idx[sel], gate[sel], ref, k)
    yref = ref["y"].copy()
    if diff.any():
        yref[diff] = nv.forward_nvfp4(ow, x64[sel][diff], k, idx=idx[sel][diff], g_x=g_x, g_h=g_h)["y"]
    return check_y(y[sel], yref, Y_TOL_NVFP4)


@pytest.fixture(scope="module")
def tiny4():
    wl = inp.workload("nvfp4_tiny")
    w = inp.make_weights(wl)
    layer = make_layer(wl, w, device_weights(w), inp.workload("nvfp4_mid").tokens)
    yield wl, w, layer
    layer.close()


def test_nvfp4_weight_bytes_small(tiny4):
    wl, w, layer = tiny4
    for e in range(wl.shape.n_experts):
        _check_weight_bytes(layer, w, 0, e)
        _check_weight_bytes(layer, w, 1, e)
    _check_weight_bytes(layer, w, 2, 0)
    _check_weight_bytes(layer, w, 3, 0)


def test_nvfp4_small_decode_shape_parity(tiny4):
    wl, w, layer = tiny4
    rel = _compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k)
    print(f"nvfp4 tiny: max|err|/RMS {rel:.3g}")


def test_nvfp4_small_prefill_shape_parity(tiny4):
    _, w, layer = tiny4
    wl = inp.workload("nvfp4_mid")
    rel = _compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k)
    print(f"nvfp4 mid: max|err|/RMS {rel:.3g}")


@pytest.mark.parametrize("t", [1, 3, 17])
def test_nvfp4_small_ragged_tokens(tiny4, t):
    wl, w, layer = tiny4
    _compare_nvfp4(layer, w, inp.make_x(inp.workload("nvfp4_mid"), tokens=t), wl.shape.top_k)


@pytest.fixture(scope="module")
def super4():
    wl = inp.workload("decode_nvfp4")
    w = host_weights("decode")
    layer = make_layer(wl, w, device_weights(w), inp.workload("prefill_nvfp4").tokens)
    yield wl, w, layer
    layer.close()
    torch.cuda.empty_cache()


def test_nvfp4_super_weight_bytes_sampled(super4):
    _, w, layer = super4
    for e in (0, 137, 511):
        _check_weight_bytes(layer, w, 0, e)
        _check_weight_bytes(layer, w, 1, e)
    _check_weight_bytes(layer, w, 2, 0)
    _check_weight_bytes(layer, w, 3, 0)


def test_nvfp4_decode_sampled_parity(super4):
    wl, w, layer = super4
    rel = _compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k, tokens=[0, 101, 255])
    print(f"nvfp4 decode: max|err|/RMS {rel:.3g}")


def test_nvfp4_prefill_sampled_parity(super4):
    _, w, layer = super4
    wl = inp.workload("prefill_nvfp4")
    rel = _compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k, tokens=[0, 9000, wl.tokens - 1])
    print(f"nvfp4 prefill: max|err|/RMS {rel:.3g}")
