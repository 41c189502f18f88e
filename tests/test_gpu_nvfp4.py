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
from lmoe_testlib import (check_weight_bytes, compare_nvfp4, device_weights, host_weights, make_layer,
                          pack_codes)

pytestmark = pytest.mark.gpu


_pack = pack_codes
_check_weight_bytes = check_weight_bytes
_compare_nvfp4 = compare_nvfp4


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


# ------------------------------------------------------------------------------------------------
# per-block MSE weight scales (lmoe_config.weight_scale = LMOE_WSCALE_MSE)
# ------------------------------------------------------------------------------------------------
@pytest.fixture(scope="module")
def tiny4_mse():
    wl = inp.workload("nvfp4_tiny")
    w = host_weights("nvfp4_tiny")
    layer = make_layer(wl, w, device_weights(w), inp.workload("nvfp4_mid").tokens, weight_scale="mse")
    yield wl, w, layer
    layer.close()


def test_nvfp4_mse_weight_bytes_small(tiny4_mse):
    wl, w, layer = tiny4_mse
    for e in range(wl.shape.n_experts):
        check_weight_bytes(layer, w, 0, e, quantize=nv.quantize_mse)
        check_weight_bytes(layer, w, 1, e, quantize=nv.quantize_mse)
    check_weight_bytes(layer, w, 2, 0, quantize=nv.quantize_mse)
    check_weight_bytes(layer, w, 3, 0, quantize=nv.quantize_mse)


def test_nvfp4_mse_parity_small(tiny4_mse):
    wl, w, layer = tiny4_mse
    compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k, weight_quantize=nv.quantize_mse)
    mid = inp.workload("nvfp4_mid")
    compare_nvfp4(layer, w, inp.make_x(mid), mid.shape.top_k, weight_quantize=nv.quantize_mse)


def test_nvfp4_mse_lowers_weight_error_small(tiny4_mse):
    """The searched scales reconstruct the weights more closely than the amax rule."""
    _, w, layer = tiny4_mse
    src = inp.bf16_bits_to_f32(w.w1[0])
    codes, scales, g = layer.export_nvfp4(0, 0)
    full = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    full[:, 0::2], full[:, 1::2] = codes & 15, codes >> 4
    e_mse = ((nv.dequantize(full, scales, g) - src) ** 2).sum()
    e_amax = ((nv.qdq(src) - src) ** 2).sum()
    assert e_mse < e_amax


def test_nvfp4_mse_super_sampled(super4):
    wl, w, _ = super4
    layer = make_layer(wl, w, device_weights(w), wl.tokens, weight_scale="mse")
    try:
        for e in (0, 511):
            check_weight_bytes(layer, w, 0, e, quantize=nv.quantize_mse)
            check_weight_bytes(layer, w, 1, e, quantize=nv.quantize_mse)
        rel = compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k, tokens=[255],
                            weight_quantize=nv.quantize_mse)
        print(f"nvfp4 mse decode: max|err|/RMS {rel:.3g}")
    finally:
        layer.close()
        torch.cuda.empty_cache()
