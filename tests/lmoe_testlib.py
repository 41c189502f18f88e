"""Helpers shared by the GPU parity tests: upload of seeded inputs, the library handle, and the
comparison rules (routing bit-exact except at logit near-ties, y within 2e-2 x RMS(y) for bf16)."""
from __future__ import annotations

import functools

import numpy as np
import torch

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo

NEAR_TIE_EPS = 1e-5       # logit gap below which routing may legitimately differ
Y_TOL_BF16 = 2e-2         # max |y_gpu - y_oracle| <= Y_TOL * RMS(y_oracle)
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
    d = {k: to_dev(getattr(w, k), dt) for k in ("w_router", "w_down", "w_up", "w1", "w2", "ws1", "ws2")}
    d["b_router"] = None if w.b_router is None else to_dev(w.b_router, "f32")
    return d


def make_layer(wl: inp.Workload, w: inp.LayerWeights, dev: dict, max_tokens: int, router_bias=None):
    import latentmoe_expert_layer_b200 as lm
    rb = wl.router_bias if router_bias is None else router_bias
    layer = lm.LatentMoE(wl.shape, max_tokens, precision=wl.precision, router_bias=rb)
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
