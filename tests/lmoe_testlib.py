"""Helpers shared by the GPU parity tests: upload of seeded inputs, the library handle, and the
comparison rules (routing bit-exact except at logit near-ties, y within 2e-2 x RMS(y) for bf16)."""
from __future__ import annotations

import functools

import numpy as np
import torch

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo
from oracle import nvfp4 as nv

NEAR_TIE_EPS = 1e-5       # logit gap below which routing may legitimately differ
Y_TOL_BF16 = 2e-2         # max |y_gpu - y_oracle| <= Y_TOL * RMS(y_oracle)
Y_TOL_NVFP4 = 5e-2        # the same against the oracle's NVFP4 forward
GATE_TOL = 1e-5           # |g_gpu - g_oracle| on tokens routed identically


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return inp.bf16_bits_to_f32(t.detach().view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


@functools.lru_cache(maxsize=2)
def host_weights(weight_seed_workload: str) -> inp.LayerWeights:
    return inp.make_weights(inp.workload(weight_seed_workload))


def device_weights(w: inp.LayerWeights) -> dict:
    dt = w.dtype
    d = {k: to_dev(getattr(w, k), dt) if getattr(w, k).size else None
         for k in ("w_router", "w_down", "w_up", "w1", "w2", "ws1", "ws2")}
    d["b_router"] = None if w.b_router is None else to_dev(w.b_router, "f32")
    return d


def make_layer(wl: inp.Workload, w: inp.LayerWeights, dev: dict, max_tokens: int, router_bias=None,
               weight_scale: str = "amax"):
    import latentmoe_expert_layer_b200 as lm
    rb = wl.router_bias if router_bias is None else router_bias
    layer = lm.LatentMoE(wl.shape, max_tokens, precision=wl.precision, router_bias=rb, weight_scale=weight_scale)
    b = None
    if rb:
        b = to_dev(inp.skewed_router_bias(), "f32")
    layer.load_weights(dev["w_router"], dev["w_down"], dev["w_up"], dev["w1"], dev["w2"], dev["ws1"], dev["ws2"],
                       b_router=b)
    return layer


def oracle_weights(w: inp.LayerWeights, bias: bool) -> lo.OracleWeights:
    ow = lo.OracleWeights(w)
    if bias:
        ow.b_router = inp.skewed_router_bias().astype(np.float64)
    return ow


def check_routing(idx_gpu: np.ndarray, gate_gpu: np.ndarray, ref: dict, k: int):
    """Return (mismatched-token mask, near-tie mask).  Asserts that every token whose routing differs
    is a near-tie, and that gates agree on all identically routed tokens."""
    near = lo.near_tie_tokens(ref["logits"], k, NEAR_TIE_EPS)
    diff = np.any(idx_gpu != ref["idx"], axis=1)
    bad = diff & ~near
    assert not bad.any(), f"{bad.sum()} tokens routed differently without a near-tie, e.g. {np.nonzero(bad)[0][:5]}"
    same = ~diff
    if same.any():
        gerr = np.abs(gate_gpu[same] - ref["gate"][same]).max()
        assert gerr <= GATE_TOL, f"gate error {gerr}"
    assert np.allclose(gate_gpu.sum(axis=1), 1.0, atol=1e-5)
    return diff, near


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray, tol: float = Y_TOL_BF16) -> float:
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = float(np.abs(y_gpu - y_ref).max())
    assert err <= tol * rms, f"max |y - y_ref| = {err:.4g} > {tol} * RMS {rms:.4g}"
    return err / rms


# ------------------------------------------------------------------------------------------------
# running the layer and comparing with the oracle
# ------------------------------------------------------------------------------------------------
def run_layer(layer, x_np):
    """Forward on x (bf16 bits); returns y (float64), idx, gate as numpy; asserts a clean status."""
    x = to_dev(x_np, "bf16")
    y, idx, gate = layer.forward(x)
    torch.cuda.synchronize()
    st = layer.device_status()
    assert st == 0, f"device status {st}"
    return bf16_to_np(y), idx.cpu().numpy(), gate.cpu().numpy()


def compare_bf16(layer, ow, x_np, k, tokens=None):
    """Run the layer on x, compare (optionally only `tokens`) with the oracle; returns stats."""
    y, idx, gate = run_layer(layer, x_np)
    x64 = lo.lift(x_np, "bf16")
    sel = np.arange(x_np.shape[0]) if tokens is None else np.asarray(tokens)
    ref = lo.forward(ow, x64[sel], k)
    diff, near = check_routing(idx[sel], gate[sel], ref, k)
    yref = ref["y"].copy()
    if diff.any():
        forced = lo.forward(ow, x64[sel][diff], k, idx=idx[sel][diff])
        yref[diff] = forced["y"]
    rel = check_y(y[sel], yref)
    # router logits of the sampled tokens
    lg = layer.inspect("logits").cpu().numpy().reshape(x_np.shape[0], -1)[sel]
    lerr = float(np.abs(lg - (ref["logits"] - (0 if ow.b_router is None else ow.b_router))).max())
    return {"y": y, "idx": idx, "gate": gate, "rel_err": rel, "logit_err": lerr, "near_ties": int(near.sum()),
            "routing_diffs": int(diff.sum())}


def check_dispatch(layer, idx, n):
    """The device's grouping maps equal the oracle's grouping of the device's own routing."""
    counts, offsets, row_of, tok_of_row = lo.dispatch(idx, n)
    assert np.array_equal(layer.inspect("counts").cpu().numpy(), counts)
    assert np.array_equal(layer.inspect("offsets").cpu().numpy(), offsets)
    assert np.array_equal(layer.inspect("row_of").cpu().numpy(), row_of.reshape(-1))
    assert np.array_equal(layer.inspect("tok_of_row").cpu().numpy(), tok_of_row)


def pack_codes(codes):
    """One E2M1 code per byte -> two per byte, element 2i in the low nibble."""
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def check_weight_bytes(layer, w, which, index, quantize=None):
    """The device's quantised weight (codes, block scales, tensor scale) equals the oracle's bytes."""
    quantize = quantize or nv.quantize
    src = {0: lambda: w.w1[index], 1: lambda: w.w2[index], 2: lambda: w.ws1, 3: lambda: w.ws2}[which]()
    ref_c, ref_s, ref_g = quantize(inp.bf16_bits_to_f32(src))
    codes, scales, g = layer.export_nvfp4(which, index)
    assert g == ref_g, (which, index, g, ref_g)
    assert np.array_equal(scales, ref_s), (which, index, np.argwhere(scales != ref_s)[:5])
    assert np.array_equal(codes, pack_codes(ref_c)), (which, index, np.argwhere(codes != pack_codes(ref_c))[:5])


def compare_nvfp4(layer, w, x_np, k, tokens=None, weight_quantize=None):
    """NVFP4 layer against the oracle's NVFP4 forward; returns max|err| / RMS(y)."""
    y, idx, gate = run_layer(layer, x_np)
    ow = oracle_weights(w, False)
    x64 = lo.lift(x_np, "bf16")
    # the per-call activation scales come from the whole batch (oracle's own x and bf16 h)
    g_x = nv.tensor_scale(x64.astype(np.float32))
    g_h = nv.tensor_scale(nv.bf16_round(x64 @ ow.w_down.T).astype(np.float32))
    sel = np.arange(x_np.shape[0]) if tokens is None else np.asarray(tokens)
    kw = {} if weight_quantize is None else {"weight_quantize": weight_quantize}
    ref = nv.forward_nvfp4(ow, x64[sel], k, g_x=g_x, g_h=g_h, **kw)
    diff, near = check_routing(idx[sel], gate[sel], ref, k)
    yref = ref["y"].copy()
    if diff.any():
        yref[diff] = nv.forward_nvfp4(ow, x64[sel][diff], k, idx=idx[sel][diff], g_x=g_x, g_h=g_h, **kw)["y"]
    return check_y(y[sel], yref, Y_TOL_NVFP4)
