"""NVFP4 quantisation and the NVFP4 layer forward, in the oracle.

TEST INFRASTRUCTURE ONLY (see lmoe_oracle.py).  Shares no code with the CUDA library.

Format.  NVFP4 stores each value as an E2M1 code (1 sign, 2 exponent, 1 mantissa bit: magnitudes
0, 0.5, 1, 1.5, 2, 3, 4, 6) with two scale levels: a fine scale per 16-element block stored as
E4M3, and one fp32 scale per tensor ("Nemotron 3 Super" notes, section 3.6: a per-tensor global
scale plus per-block fine scales; "Nemotron 3 Ultra" summary, method steps: E2M1 data and the
remark that E2M1 weights carry E4M3 block scales).  The pages fix neither the block size nor the
rounding rule; this library reads them as: 16 consecutive elements along the reduction dimension
per block, round-to-nearest-even everywhere, saturating to the largest finite value.

Scale rules (all decisions in float32, the precision the kernels use):
  per-tensor     g   = amax(|W|) / 2688            (2688 = 6 * 448: E2M1 max times E4M3 max;
                                                    an all-zero tensor gets g = 1)
  per-block      s   = E4M3_rne_sat( amax_blk / (6 * g) )
  element        q   = E2M1_rne_sat( v / (s * g) )  (s decoded back to float32 first; s == 0
                                                    gives q = 0)
  dequantised    v'  = q * s * g                     (exact)
Weights (W1_e, W2_e, W_s1, W_s2) get one g per matrix per expert; optionally (quantize_mse) a
weight block's scale is searched around s for the smallest squared reconstruction error.
Activations: x and h get a dynamic g from the amax of the whole call's tensor; u and u_s (produced
inside a GEMM epilogue, before any tensor-wide amax exists) use the static g = 1.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import lmoe_oracle as lo

__all__ = [
    "E2M1_VALUES", "e2m1_encode", "e2m1_decode", "e4m3_encode", "e4m3_decode", "tensor_scale",
    "quantize", "quantize_mse", "mse_candidates", "block_sq_error", "dequantize", "qdq", "bf16_round",
    "expert_rows_nvfp4", "forward_nvfp4",
]

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
BLOCK = 16
F32 = np.float32


def e2m1_encode(r: np.ndarray) -> np.ndarray:
    """float32 -> 4-bit code (bit 3 = sign of r, bits 0-2 = magnitude index), nearest-even, saturating."""
    r = np.asarray(r, dtype=np.float32)
    a = np.abs(r).astype(np.float64)
    a = np.minimum(a, 6.0)                               # saturate to the largest finite magnitude
    hi = np.searchsorted(E2M1_VALUES, a, side="left")    # first grid point >= a
    hi = np.minimum(hi, 7)
    lo = np.where(E2M1_VALUES[hi] == a, hi, hi - 1)
    lo = np.maximum(lo, 0)
    dlo = a - E2M1_VALUES[lo]
    dhi = E2M1_VALUES[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    sign = np.signbit(r).astype(np.uint8)
    return (sign << 3 | pick.astype(np.uint8)).astype(np.uint8)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_VALUES[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_encode(s: np.ndarray) -> np.ndarray:
    """Non-negative float32 -> E4M3 byte (bias 7, no infinities, max 448), nearest-even, saturating."""
    s = np.asarray(s, dtype=np.float32).astype(np.float64)
    if np.any(s < 0) or np.any(~np.isfinite(s)):
        raise ValueError("block scales are non-negative and finite")
    s = np.minimum(s, 448.0)
    out = np.zeros(s.shape, dtype=np.uint8)
    sub = s < 2.0 ** -6
    # subnormals: m * 2^-9, m in 0..8 (m == 8 is the smallest normal 2^-6)
    m = np.rint(s[sub] / 2.0 ** -9)                     # np.rint rounds half to even
    out[sub] = np.where(m >= 8, (1 << 3), m).astype(np.uint8)
    nrm = ~sub
    if np.any(nrm):
        v = s[nrm]
        e = np.floor(np.log2(v))
        # guard log2 rounding at exact powers of two
        e = np.where(2.0 ** e > v, e - 1, e)
        e = np.where(2.0 ** (e + 1) <= v, e + 1, e)
        q = np.rint(v / 2.0 ** (e - 3))                 # 8..16 (16 = carry into next binade)
        carry = q >= 16
        e = np.where(carry, e + 1, e)
        q = np.where(carry, 8, q)
        byte = ((e + 7).astype(np.int64) << 3) | (q.astype(np.int64) - 8)
        byte = np.minimum(byte, 0x7E)                   # 0x7E = 448 (0x7F would be NaN)
        out[nrm] = byte.astype(np.uint8)
    return out


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    e = (b >> 3) & 0xF
    m = b & 7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.where(b & 0x80, -val, val)


def tensor_scale(a: np.ndarray) -> np.float32:
    """Per-tensor scale g = amax / 2688 in float32 (1 for an all-zero tensor)."""
    amax = F32(np.max(np.abs(np.asarray(a, dtype=np.float32)))) if np.size(a) else F32(0)
    if amax == 0:
        return F32(1.0)
    return F32(amax / F32(2688.0))


def quantize(a: np.ndarray, g: Optional[np.float32] = None):
    """Quantise a [rows, cols] matrix along cols in 16-element blocks.

    Returns (codes uint8 [rows, cols] one code per element, scales uint8 [rows, cols/16] E4M3
    bytes, g float32).  Values are taken as float32 (exact for bf16 inputs)."""
    a = np.asarray(a, dtype=np.float32)
    rows, cols = a.shape
    if cols % BLOCK:
        raise ValueError("reduction dimension must be a multiple of 16")
    g = tensor_scale(a) if g is None else F32(g)
    blk = a.reshape(rows, cols // BLOCK, BLOCK)
    amax_blk = np.max(np.abs(blk), axis=2)                      # float32, exact
    den6 = F32(F32(6.0) * g)
    s_f = (amax_blk / den6).astype(np.float32)                  # float32 division, RNE
    s_b = e4m3_encode(s_f)
    s_dec = e4m3_decode(s_b).astype(np.float32)                 # exact
    den = (s_dec * g).astype(np.float32)                        # float32 product, RNE
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(den[..., None] > 0, blk / den[..., None], F32(0)).astype(np.float32)
    # keep the sign of v for exact zeros produced by an all-zero block (s == 0)
    r = np.where(den[..., None] > 0, r, np.copysign(F32(0), blk)).astype(np.float32)
    codes = e2m1_encode(r).reshape(rows, cols)
    return codes, s_b, g


MSE_DOWN = 6   # candidate block scales below the amax-derived one
MSE_UP = 1     # candidate block scales above it


def mse_candidates(c0: int):
    """E4M3 codes tried for a block whose amax-derived scale code is c0, in evaluation order:
    c0 first, then c0 + 1, then c0 - 1 ... c0 - 6, kept inside the positive finite codes 1..0x7E
    (code 0 is tried only as c0 itself)."""
    out = [c0]
    for c in [c0 + k for k in range(1, MSE_UP + 1)] + [c0 - k for k in range(1, MSE_DOWN + 1)]:
        if 1 <= c <= 0x7E and c not in out:
            out.append(c)
    return out


def block_sq_error(blk: np.ndarray, s_code: int, g: np.float32) -> np.float32:
    """Sum of squared reconstruction errors of one 16-element block (float32 values) under E4M3
    block scale code s_code, every operation in float32 in element order:
        den = s * g;  q_i = E2M1(v_i / den);  d_i = (q_i * s) * g;  e_i = v_i - d_i;  acc += e_i * e_i."""
    s = F32(e4m3_decode(np.array([s_code], np.uint8))[0])
    den = F32(s * F32(g))
    blk = np.asarray(blk, np.float32)
    if den > 0:
        q = e2m1_decode(e2m1_encode((blk / den).astype(np.float32))).astype(np.float32)
    else:
        q = np.zeros_like(blk)
    d = ((q * s).astype(np.float32) * F32(g)).astype(np.float32)
    e = (blk - d).astype(np.float32)
    acc = F32(0)
    for i in range(blk.shape[0]):
        acc = F32(acc + F32(e[i] * e[i]))
    return acc


def quantize_mse(a: np.ndarray, g: Optional[np.float32] = None):
    """Like quantize(), with each block's E4M3 scale chosen by a small search ("Nemotron 3 Super"
    notes, section 4.2, name a per-block-MSE weight quantiser without defining it; this library's
    reading): among mse_candidates(c0) of the amax-derived scale c0, the first one (in that order)
    with the strictly smallest block_sq_error.  Codes are then quantize()'s rule with that scale."""
    a = np.asarray(a, dtype=np.float32)
    rows, cols = a.shape
    if cols % BLOCK:
        raise ValueError("reduction dimension must be a multiple of 16")
    _, s0, g = quantize(a, g)
    blk = a.reshape(rows, cols // BLOCK, BLOCK)
    # block_sq_error for every block at once, one candidate offset at a time (same float32 steps
    # and element order; offsets in mse_candidates' order, so the first strict minimum wins)
    c0 = s0.astype(np.int64)
    best_c = c0.copy()
    best_e = None
    for k in [0] + list(range(1, MSE_UP + 1)) + [-j for j in range(1, MSE_DOWN + 1)]:
        c = c0 + k
        valid = np.ones_like(c, dtype=bool) if k == 0 else (c >= 1) & (c <= 0x7E)
        cc = np.clip(c, 0, 0x7E).astype(np.uint8)
        s = e4m3_decode(cc).astype(np.float32)
        den = (s * g).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            r_ = np.where(den[..., None] > 0, blk / den[..., None], F32(0)).astype(np.float32)
        q = np.where(den[..., None] > 0, e2m1_decode(e2m1_encode(r_)), 0.0).astype(np.float32)
        d = ((q * s[..., None]).astype(np.float32) * g).astype(np.float32)
        e = (blk - d).astype(np.float32)
        acc = np.zeros(c0.shape, np.float32)
        for i in range(BLOCK):
            acc = (acc + (e[..., i] * e[..., i]).astype(np.float32)).astype(np.float32)
        if best_e is None:
            best_e = acc
            continue
        better = valid & (acc < best_e)
        best_c = np.where(better, c, best_c)
        best_e = np.where(better, acc, best_e)
    s_b = best_c.astype(np.uint8)
    s_dec = e4m3_decode(s_b).astype(np.float32)
    den = (s_dec * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r_ = np.where(den[..., None] > 0, blk / den[..., None], F32(0)).astype(np.float32)
    r_ = np.where(den[..., None] > 0, r_, np.copysign(F32(0), blk)).astype(np.float32)
    return e2m1_encode(r_).reshape(rows, cols), s_b, g


def dequantize(codes: np.ndarray, scales: np.ndarray, g) -> np.ndarray:
    rows, cols = codes.shape
    v = e2m1_decode(codes).reshape(rows, cols // BLOCK, BLOCK)
    s = e4m3_decode(scales)[..., None]
    return (v * s * float(g)).reshape(rows, cols)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), via float32; returns float64 values."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def qdq(a: np.ndarray, g: Optional[np.float32] = None, quantizer=None) -> np.ndarray:
    """Quantise (quantize(), or the given quantizer) then dequantise (float64 result)."""
    c, s, gg = (quantizer or quantize)(a, g)
    return dequantize(c, s, gg)


def expert_rows_nvfp4(w: "lo.OracleWeights", hq: np.ndarray, idx: np.ndarray, gate: np.ndarray, e: int,
                      weight_quantize=None):
    """Gate-weighted outputs of expert e in the NVFP4 layer for the tokens that selected it:
    g * qdq(W2_e) qdq(sqrelu(qdq(W1_e) hq), g = 1), hq being the tokens' already quantised latents.
    Returns (tokens, rows); rows is None when no token selected e."""
    tt, kk = np.nonzero(idx == e)
    if tt.size == 0:
        return tt, None
    wq = weight_quantize or quantize
    w1 = qdq(w.w1(e).astype(np.float32), quantizer=wq)
    w2 = qdq(w.w2(e).astype(np.float32), quantizer=wq)
    u = lo.sqrelu(hq[tt] @ w1.T)
    o = qdq(u.astype(np.float32), F32(1.0)) @ w2.T
    return tt, gate[tt, kk][:, None] * o


def forward_nvfp4(w: "lo.OracleWeights", x: np.ndarray, k: int, idx: Optional[np.ndarray] = None,
                  g_x: Optional[np.float32] = None, g_h: Optional[np.float32] = None, weight_quantize=None,
                  map_fn=map):
    """Layer forward with NVFP4 routed and shared experts (weights and activations); router,
    W_down and W_up stay at the device's bf16 values.

    W_down is a BF16 layer in this variant, so the latent h it produces is a BF16 tensor: h is
    rounded to bf16 (nearest even) before it is quantised for the experts.

    g_x / g_h: per-call activation scales.  They depend on the whole call's x / h, so a caller that
    evaluates a sample of tokens passes the full batch's values.
    weight_quantize: the weights' quantiser (quantize, the default, or quantize_mse).
    map_fn: how the per-expert work is mapped over the experts (see lmoe_oracle.forward); z adds the
    experts' rows in expert order either way."""
    wq = weight_quantize or quantize
    logits = lo.router_logits(x, w.w_router, w.b_router)
    if idx is None:
        idx = lo.topk(logits, k)
    gate = lo.softmax_gates(logits, idx)
    h = bf16_round(x @ w.w_down.T)
    if g_x is None:
        g_x = tensor_scale(x.astype(np.float32))
    if g_h is None:
        g_h = tensor_scale(h.astype(np.float32))
    hq = qdq(h.astype(np.float32), g_h)
    xq = qdq(x.astype(np.float32), g_x)
    one = F32(1.0)
    z = np.zeros_like(h)
    for tt, rows in map_fn(lambda e: expert_rows_nvfp4(w, hq, idx, gate, e, wq), range(w.n_experts)):
        if rows is not None:
            z[tt] += rows
    ws1 = qdq(w.ws1.astype(np.float32), quantizer=wq)
    ws2 = qdq(w.ws2.astype(np.float32), quantizer=wq)
    us = lo.sqrelu(xq @ ws1.T)
    s = qdq(us.astype(np.float32), one) @ ws2.T
    y = z @ w.w_up.T + s
    return {"y": y, "idx": idx, "gate": gate, "logits": logits, "h": h, "z": z,
            "g_x": g_x, "g_h": g_h}
