"""Ultra-width experts (m = 5120, shared-expert intermediate 10240, with Super's d = 4096 and
l = 1024) through the same library, bf16 and NVFP4, against the oracle on sampled tokens.

The wider expert changes the GEMM shapes the library sees: 40 feature tiles per expert in the up
projection, a 5120-deep reduction in the down projection (beyond the number of K stages whose
activation scales the NVFP4 kernel keeps resident, so those launches copy scales per stage), and
an 80-stage shared expert."""
import numpy as np
import pytest
import torch

import lmoe_inputs as inp
from lmoe_testlib import (check_dispatch, check_weight_bytes, compare_bf16, compare_nvfp4, device_weights,
                          make_layer, oracle_weights)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ultra():
    wl = inp.workload("ultra_decode")
    w = inp.make_weights(wl)          # not cached: 10.9 GB of bf16 weights
    dev = device_weights(w)
    layer16 = make_layer(wl, w, dev, wl.tokens)
    layer4 = make_layer(inp.workload("ultra_decode_nvfp4"), w, dev, wl.tokens)
    torch.cuda.synchronize()
    del dev
    torch.cuda.empty_cache()
    yield w, layer16, layer4
    layer16.close()
    layer4.close()
    torch.cuda.empty_cache()


def test_ultra_decode_sampled_parity_and_dispatch(ultra):
    w, layer, _ = ultra
    wl = inp.workload("ultra_decode")
    st = compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl), wl.shape.top_k, tokens=[0, 77, 130, 255])
    check_dispatch(layer, st["idx"], wl.shape.n_experts)
    print(f"ultra decode: rel err {st['rel_err']:.3g}, logit err {st['logit_err']:.3g}")


@pytest.mark.parametrize("t", [1, 37])
def test_ultra_ragged_tokens(ultra, t):
    w, layer, _ = ultra
    wl = inp.workload("ultra_decode")
    compare_bf16(layer, oracle_weights(w, False), inp.make_x(wl, tokens=t), wl.shape.top_k,
                 tokens=np.unique([0, t - 1]))


def test_ultra_nvfp4_weight_bytes_sampled(ultra):
    w, _, layer = ultra
    for e in (3, 500):
        check_weight_bytes(layer, w, 0, e)
        check_weight_bytes(layer, w, 1, e)
    check_weight_bytes(layer, w, 3, 0)


def test_ultra_nvfp4_decode_sampled_parity(ultra):
    w, _, layer = ultra
    wl = inp.workload("ultra_decode_nvfp4")
    rel = compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k, tokens=[0, 200, 255])
    print(f"ultra nvfp4 decode: max|err|/RMS {rel:.3g}")
