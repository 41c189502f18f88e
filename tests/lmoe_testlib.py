"""Helpers shared by the GPU parity tests: upload of seeded inputs, the library handle, and the
comparison rules (routing bit-exact except at logit near-ties, y within 2e-2 x RMS(y) for bf16)."""
from __future__ import annotations

import concurrent.futures
import contextlib
import functools
import os

import numpy as np
import torch

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo
from oracle import nvfp4 as nv

NEAR_TIE_EPS = 1e-5       # logit gap below which routing may legitimately differ
LOGIT_TOL = 5e-6          # max |logit_gpu - logit_oracle|: half the near-tie gap, so that a routing
                          # decision can flip only where the oracle's gap is below NEAR_TIE_EPS
Y_TOL_BF16 = 2e-2         # max |y_gpu - y_oracle| <= Y_TOL * RMS(y_oracle)
Y_TOL_NVFP4 = 5e-2        # the same against the oracle's NVFP4 forward
GATE_TOL = 1e-5           # |g_gpu - g_oracle| on tokens routed identically


# The oracle's per-expert work runs on a thread pool (numpy releases the GIL in its array loops and
# BLAS calls); the pool's map keeps the expert order, so the oracle's sums are unchanged.
_POOL = concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


@contextlib.contextmanager
def _one_blas_thread():
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:  # pragma: no cover
        yield
        return
    with threadpool_limits(1):
        yield


def oracle_forward(ow, x64, k, idx=None):
    """lo.forward with its expert loop on the thread pool."""
    with _one_blas_thread():
        return lo.forward(ow, x64, k, idx=idx, map_fn=_POOL.map)


def oracle_forward_nvfp4(ow, x64, k, idx=None, **kw):
    """nv.forward_nvfp4 with its expert loop on the thread pool."""
    with _one_blas_thread():
        return nv.forward_nvfp4(ow, x64, k, idx=idx, map_fn=_POOL.map, **kw)


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


def oracle_routing(ow, x64: np.ndarray, k: int) -> dict:
    """The oracle's router, top-K and gates for every token (cheap next to the experts)."""
    logits = lo.router_logits(x64, ow.w_router, ow.b_router)
    idx = lo.topk(logits, k)
    return {"logits": logits, "idx": idx, "gate": lo.softmax_gates(logits, idx)}


def check_logits(layer, ow, full: dict, t: int) -> float:
    """max |logit_gpu - logit_oracle| over every token (the device buffer holds the logits before the
    router bias); asserts it is below LOGIT_TOL."""
    lg = layer.inspect("logits").cpu().numpy().reshape(t, -1).astype(np.float64)
    ref = full["logits"] - (0 if ow.b_router is None else ow.b_router[None, :])
    lerr = float(np.abs(lg - ref).max())
    assert lerr < LOGIT_TOL, f"router logit error {lerr:.3g} >= {LOGIT_TOL}"
    return lerr


def compare_bf16(layer, ow, x_np, k, tokens=None):
    """Run the layer on x.  Routing (ids bit-exact away from near-ties, gates) and the router logits
    are compared with the oracle on EVERY token; y on `tokens` (all when None).  Returns stats."""
    y, idx, gate = run_layer(layer, x_np)
    x64 = lo.lift(x_np, "bf16")
    full = oracle_routing(ow, x64, k)
    diff_all, near_all = check_routing(idx, gate, full, k)
    lerr = check_logits(layer, ow, full, x_np.shape[0])
    sel = np.arange(x_np.shape[0]) if tokens is None else np.asarray(tokens)
    ref = oracle_forward(ow, x64[sel], k)
    assert np.array_equal(ref["idx"], full["idx"][sel])
    diff = diff_all[sel]
    yref = ref["y"].copy()
    if diff.any():
        forced = oracle_forward(ow, x64[sel][diff], k, idx=idx[sel][diff])
        yref[diff] = forced["y"]
    rel = check_y(y[sel], yref)
    return {"y": y, "idx": idx, "gate": gate, "rel_err": rel, "logit_err": lerr, "near_ties": int(near_all.sum()),
            "routing_diffs": int(diff_all.sum()), "tokens_routed_checked": int(x_np.shape[0]),
            "tokens_y_checked": int(sel.size)}


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


def check_weight_bytes(layer, w, which, index, quantize=None, exported=None):
    """The device's quantised weight (codes, block scales, tensor scale) equals the oracle's bytes.
    exported: the layer's export_nvfp4(which, index), when already read."""
    quantize = quantize or nv.quantize
    src = {0: lambda: w.w1[index], 1: lambda: w.w2[index], 2: lambda: w.ws1, 3: lambda: w.ws2}[which]()
    ref_c, ref_s, ref_g = quantize(inp.bf16_bits_to_f32(src))
    codes, scales, g = exported if exported is not None else layer.export_nvfp4(which, index)
    assert g == ref_g, (which, index, g, ref_g)
    assert np.array_equal(scales, ref_s), (which, index, np.argwhere(scales != ref_s)[:5])
    assert np.array_equal(codes, pack_codes(ref_c)), (which, index, np.argwhere(codes != pack_codes(ref_c))[:5])


def compare_nvfp4(layer, w, x_np, k, tokens=None, weight_quantize=None):
    """NVFP4 layer against the oracle's NVFP4 forward.  Routing and router logits on every token; y
    on `tokens` (all when None).  Returns max|err| / RMS(y)."""
    y, idx, gate = run_layer(layer, x_np)
    ow = oracle_weights(w, False)
    x64 = lo.lift(x_np, "bf16")
    full = oracle_routing(ow, x64, k)
    diff_all, _ = check_routing(idx, gate, full, k)
    check_logits(layer, ow, full, x_np.shape[0])
    # the per-call activation scales come from the whole batch (oracle's own x and bf16 h)
    g_x = nv.tensor_scale(x64.astype(np.float32))
    g_h = nv.tensor_scale(nv.bf16_round(x64 @ ow.w_down.T).astype(np.float32))
    sel = np.arange(x_np.shape[0]) if tokens is None else np.asarray(tokens)
    kw = {} if weight_quantize is None else {"weight_quantize": weight_quantize}
    ref = oracle_forward_nvfp4(ow, x64[sel], k, g_x=g_x, g_h=g_h, **kw)
    diff = diff_all[sel]
    yref = ref["y"].copy()
    if diff.any():
        yref[diff] = oracle_forward_nvfp4(ow, x64[sel][diff], k, idx=idx[sel][diff], g_x=g_x, g_h=g_h, **kw)["y"]
    return check_y(y[sel], yref, Y_TOL_NVFP4)


# ------------------------------------------------------------------------------------------------
# NVFP4 activation bytes (codes and block scales the device wrote) against the oracle's quantiser
# ------------------------------------------------------------------------------------------------
def act_tile_rows(t: int, k: int, n: int) -> int:
    """Token-tile rows of the NVFP4 GEMM variant a forward of t tokens uses (include/lmoe.h)."""
    return 64 if t * k <= 48 * n else 192


def act_sf_bytes(buf: np.ndarray, tiles: np.ndarray, rows_in_tile: np.ndarray, kdim: int, tile_rows: int,
                 rep: int = 0) -> np.ndarray:
    """E4M3 block scales [rows, kdim / 16] read from tile-local 512-byte atoms, the layout
    include/lmoe.h gives for the LMOE_BUF_*_SF buffers (copy `rep` of replicated atoms)."""
    nra = (tile_rows + 127) // 128
    reps = 4 if tile_rows == 192 else 1
    stages = (kdim + 255) // 256
    kb = np.arange(kdim // 16)[None, :]
    st, ka, s = kb >> 4, (kb >> 2) & 3, kb & 3
    tl = np.asarray(tiles, np.int64)[:, None]
    j = np.asarray(rows_in_tile, np.int64)[:, None]
    off = (((((tl * stages + st) * 4 + ka) * nra + (j >> 7)) * reps + rep) * 512 + (j & 31) * 16 +
           ((j & 127) >> 5) * 4 + s)
    return buf[off]


def grouped_tiles(counts: np.ndarray, tile_rows: int):
    """Token tile and row-in-tile of every grouped row: tiles restart at each expert's first row."""
    counts = np.asarray(counts, np.int64)
    ntile = (counts + tile_rows - 1) // tile_rows
    tile0 = np.concatenate([[0], np.cumsum(ntile)[:-1]])
    offsets = np.concatenate([[0], np.cumsum(counts)[:-1]])
    e = np.repeat(np.arange(counts.size), counts)
    local = np.arange(int(counts.sum())) - offsets[e]
    return tile0[e] + local // tile_rows, local % tile_rows


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Two E2M1 codes per byte (element 2i low nibble) -> one code per byte."""
    out = np.empty((packed.shape[0], packed.shape[1] * 2), np.uint8)
    out[:, 0::2], out[:, 1::2] = packed & 15, packed >> 4
    return out


E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
_E4M3_VALUES = nv.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
E4M3_MIDPOINTS = (_E4M3_VALUES[1:] + _E4M3_VALUES[:-1]) / 2


def check_act_bytes(v: np.ndarray, g, codes_dev, scales_dev, code_tol: float = 0.0, scale_rtol: float = 0.0,
                    excuse_blocks: np.ndarray = None) -> dict:
    """Compare the device's NVFP4 bytes of an activation with nv.quantize(v, g).

    v [rows, K] are the oracle's values, codes_dev [rows, K] (one code per byte) and scales_dev
    [rows, K / 16] the device's.  A block whose bytes differ must be explained: its scale decision
    amax / (6 g) lies within relative scale_rtol of an E4M3 rounding midpoint, or (scale equal) each
    differing code's scaled value v / (s g) lies within code_tol of an E2M1 rounding midpoint, or
    the block is in excuse_blocks (a boolean [rows, K / 16] of blocks whose inputs legitimately
    differ).  With zero tolerances and no excuses the bytes must be identical.  Returns counts."""
    ref_c, ref_s, gg = nv.quantize(v.astype(np.float32), g)
    rows, kdim = ref_c.shape
    nb = kdim // 16
    dc = (codes_dev != ref_c).reshape(rows, nb, 16)
    ds = scales_dev != ref_s
    bad_blocks = ds | dc.any(axis=2)
    explained = np.zeros_like(bad_blocks)
    if excuse_blocks is not None:
        explained |= excuse_blocks & bad_blocks
    blk = v.reshape(rows, nb, 16).astype(np.float32)
    amax = np.abs(blk).max(axis=2).astype(np.float64)
    sdec = amax / (6.0 * float(gg))
    if ds.any() and scale_rtol > 0:
        d = np.abs(sdec[:, :, None] - E4M3_MIDPOINTS[None, None, :]).min(axis=2)
        explained |= ds & (d <= scale_rtol * np.maximum(sdec, 1e-30))
    code_only = bad_blocks & ~ds & ~explained
    if code_only.any() and code_tol > 0:
        s_ref = nv.e4m3_decode(ref_s).astype(np.float64)
        r = np.abs(blk.astype(np.float64)) / np.maximum(s_ref[:, :, None] * float(gg), 1e-300)
        near = np.abs(r[..., None] - E2M1_MIDPOINTS).min(axis=3) <= code_tol
        ok = np.all(~dc | near, axis=2)
        explained |= code_only & ok
    unexplained = bad_blocks & ~explained
    assert not unexplained.any(), (f"{int(unexplained.sum())} of {rows * nb} blocks differ away from a rounding "
                                   f"decision, e.g. {np.argwhere(unexplained)[:4].tolist()}")
    return {"blocks": rows * nb, "differing_blocks": int(bad_blocks.sum()), "scale_mismatches": int(ds.sum()),
            "code_mismatches": int(dc.sum())}
