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
from lmoe_testlib import (_POOL, act_sf_bytes, act_tile_rows, bf16_to_np, check_act_bytes, check_weight_bytes,
                          compare_nvfp4, device_weights, grouped_tiles, host_weights, make_layer, oracle_weights,
                          run_layer, unpack_codes)

pytestmark = pytest.mark.gpu

# Device activations that come out of an fp32 GEMM accumulator (u, u_s) carry its accumulation error
# (about 1e-5 relative, measured on the router GEMM), so their NVFP4 decisions may differ from the
# oracle's exactly where the value sits at a rounding decision: a scaled element v / (s g) within
# CODE_TOL of an E2M1 midpoint (its worst-case drift is ~2e-4 on the 0..6 grid), or a block scale
# decision amax / (6 g) within relative SCALE_RTOL of an E4M3 midpoint.  x and h, which enter the
# quantiser as bf16 values, must give identical bytes.
CODE_TOL = 1e-3
SCALE_RTOL = 1e-4


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
        check_weight_bytes(layer, w, 0, e)
        check_weight_bytes(layer, w, 1, e)
    check_weight_bytes(layer, w, 2, 0)
    check_weight_bytes(layer, w, 3, 0)


def test_nvfp4_small_decode_shape_parity(tiny4):
    wl, w, layer = tiny4
    rel = compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k)
    print(f"nvfp4 tiny: max|err|/RMS {rel:.3g}")


def test_nvfp4_small_prefill_shape_parity(tiny4):
    _, w, layer = tiny4
    wl = inp.workload("nvfp4_mid")
    rel = compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k)
    print(f"nvfp4 mid: max|err|/RMS {rel:.3g}")


@pytest.mark.parametrize("t", [1, 3, 17])
def test_nvfp4_small_ragged_tokens(tiny4, t):
    wl, w, layer = tiny4
    compare_nvfp4(layer, w, inp.make_x(inp.workload("nvfp4_mid"), tokens=t), wl.shape.top_k)


@pytest.fixture(scope="module")
def super4():
    wl = inp.workload("decode_nvfp4")
    w = host_weights("decode")
    layer = make_layer(wl, w, device_weights(w), inp.workload("prefill_nvfp4").tokens)
    yield wl, w, layer
    layer.close()
    torch.cuda.empty_cache()


def test_nvfp4_super_weight_bytes_sampled(super4):
    """32 experts spread over the 512 (W1 and W2 each), and the shared expert."""
    _, w, layer = super4
    experts = list(range(0, 512, 16))
    experts[-1] = 511
    exported = {(which, e): layer.export_nvfp4(which, e) for e in experts for which in (0, 1)}

    def one(key):
        check_weight_bytes(layer, w, key[0], key[1], exported=exported[key])
        return key

    assert len(list(_POOL.map(one, list(exported)))) == 2 * len(experts)
    check_weight_bytes(layer, w, 2, 0)
    check_weight_bytes(layer, w, 3, 0)


def test_nvfp4_decode_full_parity(super4):
    """Every token of the decode batch."""
    wl, w, layer = super4
    rel = compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k)
    print(f"nvfp4 decode: max|err|/RMS {rel:.3g} on all {wl.tokens} tokens")


def test_nvfp4_prefill_sampled_parity(super4):
    """64 tokens, one in each 256-token stretch of the batch (so every 192-row token tile region of
    the dense tensors is visited), routing and logits on all 16384."""
    _, w, layer = super4
    wl = inp.workload("prefill_nvfp4")
    tokens = np.unique(np.concatenate([[0, wl.tokens - 1], np.arange(64) * 256 + (np.arange(64) * 37) % 256]))
    rel = compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k, tokens=tokens)
    print(f"nvfp4 prefill: max|err|/RMS {rel:.3g} on {tokens.size} tokens")


def _activation_bytes(layer, w, wl, x_np, grouped_rows=None, dense_rows=None, u_experts=None):
    """Device NVFP4 activation bytes against the oracle's quantiser after one forward on x:
    x (exact), the grouped h rows (exact, except blocks whose bf16 h input differs between the
    device's W_down GEMM and the oracle's rounded fp64 product), u_s and u (within the rounding-
    decision tolerances).  Also the per-call tensor scales g_x, g_h.  Returns the counts."""
    s = wl.shape
    t = x_np.shape[0]
    tk = t * s.top_k
    R = act_tile_rows(t, s.top_k, s.n_experts)
    run_layer(layer, x_np)
    ow = oracle_weights(w, False)
    x64 = lo.lift(x_np, "bf16")
    g_x = nv.tensor_scale(x64.astype(np.float32))
    h_or = nv.bf16_round(x64 @ ow.w_down.T)
    g_h = nv.tensor_scale(h_or.astype(np.float32))
    act = layer.inspect("act_scale").cpu().numpy()
    assert act[0] == g_x and act[1] == g_h, (act, g_x, g_h)
    out = {}
    dense = np.arange(t) if dense_rows is None else np.asarray(dense_rows)
    xq = unpack_codes(layer.inspect("xq").cpu().numpy()[: t * s.d // 2].reshape(t, s.d // 2))
    xsf = act_sf_bytes(layer.inspect("x_sf").cpu().numpy(), np.arange(t) // R, np.arange(t) % R, s.d, R)
    out["x"] = check_act_bytes(x64, g_x, xq, xsf)
    counts = layer.inspect("counts").cpu().numpy()
    tok = layer.inspect("tok_of_row").cpu().numpy()
    tiles, jrow = grouped_tiles(counts, R)
    rows = np.arange(tk) if grouped_rows is None else np.asarray(grouped_rows)
    hq = unpack_codes(layer.inspect("hq").cpu().numpy().reshape(-1, s.latent // 2)[rows])
    hsf = act_sf_bytes(layer.inspect("h_sf").cpu().numpy(), tiles[rows], jrow[rows], s.latent, R)
    h_dev = bf16_to_np(layer.inspect("h").view(torch.bfloat16)).reshape(t, s.latent)
    h_differs = (h_dev != h_or).reshape(t, s.latent // 16, 16).any(axis=2)
    out["h"] = check_act_bytes(h_or[tok[rows]], g_h, hq, hsf, excuse_blocks=h_differs[tok[rows]])
    out["h_input_blocks_differing"] = int(h_differs.sum())
    # u_s = sqrelu(qdq(W_s1) qdq(x)) quantised with g = 1
    xq_or = nv.qdq(x64[dense].astype(np.float32), g_x)
    us_or = lo.sqrelu(xq_or @ nv.qdq(ow.ws1.astype(np.float32)).T)
    usq = unpack_codes(layer.inspect("usq").cpu().numpy()[: t * s.shared_ffn // 2].reshape(t, -1)[dense])
    ussf = act_sf_bytes(layer.inspect("us_sf").cpu().numpy(), dense // R, dense % R, s.shared_ffn, R)
    out["u_s"] = check_act_bytes(us_or, np.float32(1.0), usq, ussf, CODE_TOL, SCALE_RTOL)
    # u = sqrelu(qdq(W1_e) qdq(h)) of the grouped rows of the given experts
    if u_experts is not None:
        offs = layer.inspect("offsets").cpu().numpy()
        hq_or = nv.qdq(h_or.astype(np.float32), g_h)
        uq_all = layer.inspect("uq").cpu().numpy().reshape(-1, s.expert_ffn // 2)
        usf_all = layer.inspect("u_sf").cpu().numpy()
        stats = []
        for e in u_experts:
            r = np.arange(offs[e], offs[e + 1])
            if r.size == 0:
                continue
            u_or = lo.sqrelu(hq_or[tok[r]] @ nv.qdq(ow.w1(e).astype(np.float32)).T)
            st = check_act_bytes(u_or, np.float32(1.0), unpack_codes(uq_all[r]),
                                 act_sf_bytes(usf_all, tiles[r], jrow[r], s.expert_ffn, R), CODE_TOL, SCALE_RTOL,
                                 excuse_blocks=np.repeat(h_differs[tok[r]].any(axis=1)[:, None],
                                                         s.expert_ffn // 16, axis=1))
            stats.append(st)
        out["u"] = {k: sum(st[k] for st in stats) for k in stats[0]}
    return out


def test_nvfp4_activation_bytes_small(tiny4):
    """Both GEMM variants (64- and 192-row token tiles) on the small NVFP4 layer, every row."""
    wl, w, layer = tiny4
    experts = range(wl.shape.n_experts)
    for name in ("nvfp4_tiny", "nvfp4_mid"):
        st = _activation_bytes(layer, w, inp.workload(name), inp.make_x(inp.workload(name)), u_experts=experts)
        print(f"{name} activation bytes: {st}")


def test_nvfp4_activation_bytes_decode(super4):
    wl, w, layer = super4
    st = _activation_bytes(layer, w, wl, inp.make_x(wl), u_experts=[0, 1, 137, 511])
    print(f"nvfp4 decode activation bytes: {st}")


def test_nvfp4_activation_bytes_prefill(super4):
    """x on all 16384 tokens; h on 8192 sampled grouped rows; u_s on 256 sampled tokens; u on 2 experts."""
    _, w, layer = super4
    wl = inp.workload("prefill_nvfp4")
    rng = np.random.default_rng(3)
    st = _activation_bytes(layer, w, wl, inp.make_x(wl),
                           grouped_rows=np.sort(rng.choice(wl.tokens * wl.shape.top_k, 8192, replace=False)),
                           dense_rows=np.sort(rng.choice(wl.tokens, 256, replace=False)), u_experts=[0, 300])
    print(f"nvfp4 prefill activation bytes: {st}")


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
        rel = compare_nvfp4(layer, w, inp.make_x(wl), wl.shape.top_k, tokens=[0, 128, 255],
                            weight_quantize=nv.quantize_mse)
        print(f"nvfp4 mse decode: max|err|/RMS {rel:.3g}")
    finally:
        layer.close()
        torch.cuda.empty_cache()
