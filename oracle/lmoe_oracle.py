"""fp64 CPU oracle of the LatentMoE layer forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke entry point and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and never calls it.

What it computes, per token t (x in R^d), written out plainly:

  1. router logits     l_e = sum_j x_j W_r[e, j] + b_e                  (gating network runs in the
                                                                         full dimension d: "Nemotron 3
                                                                         Super" notes, section 3.2,
                                                                         last paragraph)
  2. top-K             S = the K largest l_e, ordered by (l desc, e asc) (architecture table,
                                                                         section 3.1: top-K = 22 of 512)
  3. gate              g_k = softmax over the K selected logits           (the pages do not fix the
                                                                         normalisation; softmax over
                                                                         the selected K is the reading
                                                                         this library takes)
  4. latent            h = W_down x,  W_down in R^{l x d}                 (section 3.2, first paragraph)
  5. routed experts    z = sum_k g_k W2_{S_k} sqrelu(W1_{S_k} h)          (experts run in the latent
                                                                         space, l -> m -> l; squared
                                                                         ReLU, non-gated, no bias)
  6. output            y = W_up z + W_s2 sqrelu(W_s1 x),  W_up in R^{d x l} (section 3.2; the shared
                                                                         expert runs in full d)
  A layer given without W_down and W_up is the standard MoE of the same section: h = x and
  y = z + W_s2 sqrelu(W_s1 x).

Everything is float64 numpy; weights arrive as the exact values the device consumes (bf16 bit
patterns or float32) and are lifted losslessly.  Per-expert work loops over experts, lifting one
expert at a time, so the Super shape (2.9 G parameters) never needs more than a few hundred MB.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

import lmoe_inputs as inp

__all__ = [
    "lift", "OracleWeights", "router_logits", "topk", "softmax_gates", "sqrelu", "dispatch",
    "near_tie_tokens", "expert_rows", "forward",
]


def lift(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 copy of a device tensor (uint16 bf16 bits, or float32)."""
    if dtype == "bf16":
        return inp.bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


class OracleWeights:
    """float64 view of a layer's weights as the library consumes them.

    For float32 input weights the library converts every matrix except the router to bf16 at
    load time (round to nearest even); the oracle is given those same rounded values.
    """

    def __init__(self, w: "inp.LayerWeights"):
        self.src = w
        as_dev = (lambda a: lift(inp.f32_to_bf16_bits(a), "bf16")) if w.dtype == "f32" else \
                 (lambda a: lift(a, "bf16"))
        self._as_dev = as_dev
        self.w_router = lift(w.w_router, w.dtype)          # fp32 router stays fp32
        self.b_router = None if w.b_router is None else np.asarray(w.b_router, np.float32).astype(np.float64)
        self.w_down = as_dev(w.w_down)
        self.w_up = as_dev(w.w_up)
        self.ws1 = as_dev(w.ws1)
        self.ws2 = as_dev(w.ws2)
        self.n_experts = w.w_router.shape[0]

    def w1(self, e: int) -> np.ndarray:
        return self._as_dev(self.src.w1[e])

    def w2(self, e: int) -> np.ndarray:
        return self._as_dev(self.src.w2[e])


def router_logits(x: np.ndarray, w_router: np.ndarray, b_router: Optional[np.ndarray] = None) -> np.ndarray:
    """l[t, e] = x[t, :] . W_r[e, :] (+ b[e]).  Shapes x [T, d], W_r [N, d] -> [T, N]."""
    l = x @ w_router.T
    if b_router is not None:
        l = l + b_router[None, :]
    return l


def topk(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, ordered by value descending, ties to the lower
    expert index.  Returns int32 [T, k]."""
    # a stable ascending sort of -logit keeps equal logits in index order
    order = np.argsort(-logits, axis=1, kind="stable")
    return np.ascontiguousarray(order[:, :k]).astype(np.int32)


def softmax_gates(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g[t, k] = exp(l[t, idx[t,k]] - max) / sum_k' exp(l[t, idx[t,k']] - max)."""
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    e = np.exp(sel - sel.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def sqrelu(v: np.ndarray) -> np.ndarray:
    """Squared ReLU, elementwise: max(v, 0)^2."""
    r = np.maximum(v, 0.0)
    return r * r


def dispatch(idx: np.ndarray, n_experts: int):
    """Group the (token, slot) assignments by expert.

    counts[e]      number of (t, k) with idx[t, k] == e
    offsets[e]     exclusive prefix sum of counts (length N + 1)
    row_of[t, k]   offsets[e] + (number of earlier assignments to e in (t, k) row-major order)
    tok_of_row[r]  the token whose assignment sits at row r
    All int32; the grouping is stable, so every output is uniquely defined.
    """
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    np.cumsum(counts, out=offsets[1:])
    order = np.argsort(flat, kind="stable")
    row_of = np.empty_like(flat)
    row_of[order] = np.arange(flat.size)
    tok_of_row = (order // idx.shape[1]).astype(np.int64)
    return (counts.astype(np.int32), offsets.astype(np.int32),
            row_of.reshape(idx.shape).astype(np.int32), tok_of_row.astype(np.int32))


def near_tie_tokens(logits: np.ndarray, k: int, eps: float) -> np.ndarray:
    """Boolean [T]: token whose selection or order is decided by a logit gap below eps.

    A token is a near-tie when the gap between the K-th and (K+1)-th largest logit is below eps
    (set membership could flip) or when any two adjacent selected logits differ by less than eps
    (their order could flip)."""
    s = -np.sort(-logits, axis=1)
    m = np.zeros(logits.shape[0], dtype=bool)
    if k < logits.shape[1]:
        m |= (s[:, k - 1] - s[:, k]) < eps
    if k > 1:
        m |= (np.diff(-s[:, :k], axis=1) < eps).any(axis=1)
    return m


def expert_rows(w: OracleWeights, h: np.ndarray, idx: np.ndarray, gate: np.ndarray, e: int):
    """Gate-weighted outputs g * W2_e sqrelu(W1_e h[t]) of expert e for the tokens t that selected it.
    Returns (tokens, rows [n, width of h]); rows is None when no token selected e."""
    tt, kk = np.nonzero(idx == e)
    if tt.size == 0:
        return tt, None
    u = sqrelu(h[tt] @ w.w1(e).T)
    o = u @ w.w2(e).T
    return tt, gate[tt, kk][:, None] * o


def forward(w: OracleWeights, x: np.ndarray, k: int, idx: Optional[np.ndarray] = None, map_fn=map):
    """Full layer forward in float64.

    x      [T, d] float64 (the exact bf16 values the device sees)
    k      top-K
    idx    optional forced routing [T, K] (used to re-evaluate tokens whose GPU routing differs at a
           near-tie); gates are then the softmax of the oracle's own logits at those experts.
    map_fn how the per-expert work is mapped over the experts (the built-in map, or a thread pool's
           map, which keeps the order); z adds the experts' rows in expert order either way.
    Returns dict with y [T, d], idx [T, K], gate [T, K], logits [T, N], h [T, l], z [T, l].

    A layer given without W_down / W_up (w.w_down with zero rows) is the standard MoE these replace
    ("Nemotron 3 Super" notes, section 3.2): the experts run on x itself (d -> m -> d) and
    y = z + W_s2 sqrelu(W_s1 x).
    """
    logits = router_logits(x, w.w_router, w.b_router)
    if idx is None:
        idx = topk(logits, k)
    gate = softmax_gates(logits, idx)
    standard = w.w_down.shape[0] == 0
    h = x if standard else x @ w.w_down.T
    z = np.zeros_like(h)
    # each token selects an expert at most once, so a token appears once in an expert's rows
    for tt, rows in map_fn(lambda e: expert_rows(w, h, idx, gate, e), range(w.n_experts)):
        if rows is not None:
            z[tt] += rows
    s = sqrelu(x @ w.ws1.T) @ w.ws2.T
    y = (z if standard else z @ w.w_up.T) + s
    return {"y": y, "idx": idx, "gate": gate, "logits": logits, "h": h, "z": z}
