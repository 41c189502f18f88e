"""Seeded synthetic inputs for the LatentMoE layer (shared by the oracle side and the CUDA side).

This module holds workload definitions and random-number generation only.  It contains none of
the layer's arithmetic (no router, no top-K, no projection, no expert): it draws weights and
activations, rounds them to the dtype the device consumes, and returns plain numpy arrays.

Shapes follow the architecture table of "Nemotron 3 Super" (guokunwang.com notes, section 3.1:
model dim 4096, expert hidden 2688, shared-expert intermediate 5376, 512 experts per layer,
top-22, MoE latent dim 1024).  The LatentMoE matrices are W_down in R^{l x d} and W_up in R^{d x l}
(same notes, section 3.2).  Every weight matrix is stored row-major as [out, in].

Generation recipe (fixed, documented):
  * numpy PCG64, one child stream per tensor from SeedSequence(seed).spawn(8), and for the
    per-expert tensors W1/W2 one grandchild stream per expert (so one expert can be regenerated
    alone);
  * every matrix ~ N(0, 1/fan_in) with fan_in = its input dimension, x ~ N(0, 1);
  * values are drawn in float32 and rounded to bfloat16 (round to nearest even) when the device
    dtype is bf16.  The tiny workload keeps float32 weights (the library converts them at load;
    the oracle is handed the same bf16 rounding, except for the router which stays fp32).
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np

__all__ = [
    "LayerShape", "SUPER", "ULTRA", "STANDARD", "Workload", "WORKLOADS", "workload", "f32_to_bf16_bits", "bf16_bits_to_f32",
    "LayerWeights", "make_weights", "make_router", "make_x", "expert_weight", "skewed_router_bias",
]


@dataclasses.dataclass(frozen=True)
class LayerShape:
    d: int            # model dimension
    latent: int       # LatentMoE latent dimension l
    n_experts: int    # N
    top_k: int        # K
    expert_ffn: int   # m  (routed expert hidden)
    shared_ffn: int   # m_s (shared expert hidden)

    @property
    def expert_in(self) -> int:
        """Width the routed experts work in: l, or d for a standard MoE (latent = 0)."""
        return self.latent if self.latent else self.d

    @property
    def params(self) -> int:
        s = self
        return (s.n_experts * s.d + 2 * s.latent * s.d + 2 * s.n_experts * s.expert_ffn * s.expert_in
                + 2 * s.d * s.shared_ffn)


SUPER = LayerShape(d=4096, latent=1024, n_experts=512, top_k=22, expert_ffn=2688, shared_ffn=5376)
# Ultra-width experts: 512 experts, top-22, expert hidden 5120, shared-expert intermediate 10240
# ("Nemotron 3 Ultra" summary, core method).  That page gives neither the model dimension nor the
# latent dimension, so Super's d = 4096 and l = 1024 are kept.
ULTRA = LayerShape(d=4096, latent=1024, n_experts=512, top_k=22, expert_ffn=5120, shared_ffn=10240)
# The standard MoE with the Super layer's budget: LatentMoE turns N, K into N' = N d / l and
# K' = K d / l ("Nemotron 3 Super" notes, section 3.2), so N = 512 * 1024 / 4096 = 128 experts and
# K = 22 / 4 = 5.5, rounded to 6; experts d -> m -> d with no W_down / W_up (latent = 0).
STANDARD = LayerShape(d=4096, latent=0, n_experts=128, top_k=6, expert_ffn=2688, shared_ffn=5376)
TINY = LayerShape(d=256, latent=64, n_experts=16, top_k=4, expert_ffn=128, shared_ffn=256)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    tokens: int
    weight_seed: int
    x_seed: int
    weight_dtype: str          # "f32" (tiny) or "bf16"
    precision: str             # "bf16" or "nvfp4"
    router_bias: bool = False  # skewed workload only
    description: str = ""


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", TINY, 64, 0, 0, "f32", "bf16",
                     description="tiny LatentMoE layer T=64 d=256 l=64 N=16 K=4 m=128 m_s=256, fp32 weights"),
    "decode": Workload("decode", SUPER, 256, 1, 2, "bf16", "bf16",
                       description="Super-shaped decode/verify batch T=256 (32 sequences x 8 positions)"),
    "prefill": Workload("prefill", SUPER, 16384, 1, 3, "bf16", "bf16",
                        description="Super-shaped prefill T=16384, near-uniform expert load"),
    "decode_nvfp4": Workload("decode_nvfp4", SUPER, 256, 1, 2, "bf16", "nvfp4",
                             description="NVFP4 experts+shared expert, decode batch T=256"),
    "prefill_nvfp4": Workload("prefill_nvfp4", SUPER, 16384, 1, 3, "bf16", "nvfp4",
                              description="NVFP4 experts+shared expert, prefill T=16384"),
    # profiling case: the decode kernels' regime (~11 tokens per expert, weights streamed once) on a
    # 128-expert layer, so that a full-metric profiler capture holds ~1.5 GB on the device
    "decode_small": Workload("decode_small", dataclasses.replace(SUPER, n_experts=128), 64, 1, 2, "bf16", "bf16",
                             description="Super dims with 128 experts, T=64 (~11 tokens per expert)"),
    # profiling case: the prefill kernels' regime (~704 tokens per expert, 256-token tiles) with 128
    # experts, ~2.3 GB on the device
    "prefill_small": Workload("prefill_small", dataclasses.replace(SUPER, n_experts=128), 4096, 1, 3, "bf16", "bf16",
                              description="Super dims with 128 experts, T=4096 (~704 tokens per expert)"),
    # profiling case: the NVFP4 prefill GEMM's regime (~704 tokens per expert, 192-token tiles) with
    # 128 experts, under 1 GB on the device
    "prefill_small_nvfp4": Workload("prefill_small_nvfp4", dataclasses.replace(SUPER, n_experts=128), 4096, 1, 3,
                                    "bf16", "nvfp4",
                                    description="NVFP4 Super dims with 128 experts, T=4096 (~704 tokens per expert)"),
    # small NVFP4 layers: several 128-row tiles, a ragged 256-element K stage (m = 384), both the
    # decode-sized (~10 tokens per expert) and the prefill-sized (~256 per expert) GEMM shapes
    "nvfp4_tiny": Workload("nvfp4_tiny", LayerShape(512, 256, 16, 4, 384, 512), 40, 7, 8, "bf16", "nvfp4",
                           description="NVFP4 layer d=512 l=256 N=16 K=4 m=384 m_s=512, T=40"),
    "nvfp4_mid": Workload("nvfp4_mid", LayerShape(512, 256, 16, 4, 384, 512), 1024, 7, 9, "bf16", "nvfp4",
                          description="NVFP4 layer d=512 l=256 N=16 K=4 m=384 m_s=512, T=1024"),
    "ultra_decode": Workload("ultra_decode", ULTRA, 256, 5, 2, "bf16", "bf16",
                             description="Ultra-width experts (m=5120, m_s=10240; d=4096, l=1024), decode T=256"),
    "ultra_decode_nvfp4": Workload("ultra_decode_nvfp4", ULTRA, 256, 5, 2, "bf16", "nvfp4",
                                   description="NVFP4 Ultra-width experts, decode T=256"),
    "ultra_prefill": Workload("ultra_prefill", ULTRA, 16384, 5, 3, "bf16", "bf16",
                              description="Ultra-width experts, prefill T=16384"),
    "standard_decode": Workload("standard_decode", STANDARD, 256, 6, 2, "bf16", "bf16",
                                description="standard MoE of the Super budget (N=128, K=6, experts d->m->d, "
                                            "no W_down/W_up), decode T=256"),
    "standard_prefill": Workload("standard_prefill", STANDARD, 16384, 6, 3, "bf16", "bf16",
                                 description="standard MoE of the Super budget, prefill T=16384"),
    "skewed": Workload("skewed", SUPER, 4096, 1, 4, "bf16", "bf16", router_bias=True,
                       description="Super shape T=4096, per-expert router bias giving a capped Zipf(1.2) load"),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


# ---------------------------------------------------------------------------------------------
# dtype helpers (input preparation, not layer arithmetic)
# ---------------------------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, nearest-even; returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------------------------
# random streams
# ---------------------------------------------------------------------------------------------
_TENSORS = ("w_router", "w_down", "w_up", "w1", "w2", "ws1", "ws2", "x")


def _streams(seed: int):
    kids = np.random.SeedSequence(seed).spawn(len(_TENSORS))
    return dict(zip(_TENSORS, kids))


def _normal(ss: np.random.SeedSequence, shape, std: float) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(ss))
    a = g.standard_normal(size=shape, dtype=np.float32)
    a *= np.float32(std)
    return a


def _finish(a: np.ndarray, dtype: str) -> np.ndarray:
    return a if dtype == "f32" else f32_to_bf16_bits(a)


def expert_weight(wl: Workload, which: str, e: int) -> np.ndarray:
    """One expert's W1 [m, l] or W2 [l, m], in the device dtype (uint16 bf16 bits or float32)."""
    s = wl.shape
    ss = _streams(wl.weight_seed)[which].spawn(s.n_experts)[e]
    if which == "w1":
        return _finish(_normal(ss, (s.expert_ffn, s.expert_in), 1.0 / np.sqrt(s.expert_in)), wl.weight_dtype)
    if which == "w2":
        return _finish(_normal(ss, (s.expert_in, s.expert_ffn), 1.0 / np.sqrt(s.expert_ffn)), wl.weight_dtype)
    raise ValueError(which)


@dataclasses.dataclass
class LayerWeights:
    """All weights of one layer in the device dtype.  bf16 tensors are uint16 bit patterns."""
    w_router: np.ndarray   # [N, d]
    b_router: Optional[np.ndarray]  # [N] float32 or None
    w_down: np.ndarray     # [l, d]   ([0, d] for a standard MoE)
    w_up: np.ndarray       # [d, l]   ([d, 0] for a standard MoE)
    w1: np.ndarray         # [N, m, l] ([N, m, d] for a standard MoE)
    w2: np.ndarray         # [N, l, m] ([N, d, m] for a standard MoE)
    ws1: np.ndarray        # [m_s, d]
    ws2: np.ndarray        # [d, m_s]
    dtype: str             # "f32" or "bf16"


def make_weights(wl: Workload, threads: Optional[int] = None, experts: bool = True) -> LayerWeights:
    """Draw the full layer.  With experts=False, W1/W2 are left empty (shape [0, ...])."""
    s = wl.shape
    st = _streams(wl.weight_seed)
    f = lambda name, shape, fan: _finish(_normal(st[name], shape, 1.0 / np.sqrt(fan)), wl.weight_dtype)
    # the router keeps fp32 in the tiny (fp32) workload, bf16 otherwise
    w_router = f("w_router", (s.n_experts, s.d), s.d)
    w_down = f("w_down", (s.latent, s.d), s.d)
    w_up = f("w_up", (s.d, s.latent), s.latent) if s.latent else w_down.reshape(s.d, 0)
    ws1 = f("ws1", (s.shared_ffn, s.d), s.d)
    ws2 = f("ws2", (s.d, s.shared_ffn), s.shared_ffn)
    dt = np.float32 if wl.weight_dtype == "f32" else np.uint16
    n = s.n_experts if experts else 0
    w1 = np.empty((n, s.expert_ffn, s.expert_in), dtype=dt)
    w2 = np.empty((n, s.expert_in, s.expert_ffn), dtype=dt)
    if n:
        threads = threads or min(32, os.cpu_count() or 1)

        def fill(e):
            w1[e] = expert_weight(wl, "w1", e)
            w2[e] = expert_weight(wl, "w2", e)

        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(n)))
    b = skewed_router_bias() if wl.router_bias else None
    return LayerWeights(w_router, b, w_down, w_up, w1, w2, ws1, ws2, wl.weight_dtype)


def make_router(wl: Workload) -> np.ndarray:
    """Only the router weight W_r [N, d] (device dtype), without drawing the rest of the layer."""
    s = wl.shape
    return _finish(_normal(_streams(wl.weight_seed)["w_router"], (s.n_experts, s.d), 1.0 / np.sqrt(s.d)),
                   wl.weight_dtype)


def make_x(wl: Workload, tokens: Optional[int] = None) -> np.ndarray:
    """Activations x [T, d] as bf16 bits (every workload feeds bf16 activations to the layer)."""
    t = wl.tokens if tokens is None else tokens
    a = _normal(_streams(wl.x_seed)["x"], (wl.tokens, wl.shape.d), 1.0)
    return f32_to_bf16_bits(a[:t])


_BIAS_FILE = os.path.join(os.path.dirname(__file__), "skewed_router_bias_f32.txt")


def skewed_router_bias() -> np.ndarray:
    """Per-expert router bias of the skewed workload (float32 [512]).

    The values were fitted once, offline, so that the top-22 load of the skewed workload's x
    follows a capped Zipf(1.2) profile with 32 idle experts; the fitting script and its rule live
    with the oracle.  Stored as float32 hex so the bits round-trip exactly.
    """
    with open(_BIAS_FILE) as fh:
        vals = [int(tok, 16) for line in fh for tok in line.split() if not line.startswith("#")]
    return np.array(vals, dtype=np.uint32).view(np.float32)
