"""Pins of the oracle's NVFP4 layer composition (oracle/nvfp4.py forward_nvfp4), CPU only.

The NVFP4 format functions are pinned in test_oracle_pins.py.  Here the question is how the layer
uses them: which tensors are quantised (x for the shared expert, the bf16-rounded h for the routed
experts, u and u_s re-quantised, the four expert weight matrices), with which tensor scale (dynamic
g_x and g_h from the whole batch, g = 1 for u and u_s), and in which order.  Three pins:

1. Closed form: on a layer built so that every quantised tensor is exactly representable in NVFP4
   (each 16-element block holds E2M1 codes times a power-of-two E4M3 scale times an exact tensor
   scale, and u, u_s come out representable too), quantise-then-dequantise is the identity, so the
   NVFP4 forward must equal the plain bf16 forward lmoe_oracle.forward.
2. Restatement: a per-token scalar loop written from the format's definition (round to the nearest
   grid point by brute-force search over the 8 E2M1 magnitudes and the 127 E4M3 values, ties to the
   even code; fp32 decisions) must reproduce forward_nvfp4 on a random layer.
3. Planted mistakes: the same restatement with u not re-quantised, with h quantised under g_x, or
   with h not rounded to bf16 must each differ from forward_nvfp4 on that layer, so a slip of that
   kind in the oracle would fail pin 2.
"""
import math
import struct

import numpy as np
import pytest

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo
from oracle import nvfp4 as nv

F32 = np.float32


# ------------------------------------------------------------------------------------------------
# scalar NVFP4, written from the format definition (brute-force nearest grid point)
# ------------------------------------------------------------------------------------------------
E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e4m3_value(code: int) -> float:
    e, m = code >> 3, code & 7
    return m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_GRID = [_e4m3_value(c) for c in range(0x7F)]   # codes 0..0x7E (0x7F is NaN)


def _nearest(a: float, grid) -> float:
    """The grid value nearest to a (a clamped into the grid's range); on a tie, the even index."""
    a = min(a, grid[-1])
    best_i, best_d = 0, abs(a - grid[0])
    for i in range(1, len(grid)):
        dd = abs(a - grid[i])
        if dd < best_d or (dd == best_d and i % 2 == 0):
            best_i, best_d = i, dd
    return grid[best_i]


def scalar_tensor_scale(values) -> float:
    amax = max((abs(float(F32(v))) for v in values), default=0.0)
    return 1.0 if amax == 0 else float(F32(F32(amax) / F32(2688.0)))


def scalar_qdq_block(vals, g: float):
    """Quantise-dequantise 16 values with tensor scale g: E4M3 block scale of amax / (6 g), then each
    element's E2M1 value of v / (s g); every decision on fp32 values."""
    g32 = F32(g)
    amax = max(abs(float(F32(v))) for v in vals)
    s = _nearest(float(F32(F32(amax) / F32(F32(6.0) * g32))), E4M3_GRID)
    den = F32(F32(s) * g32)
    if den == 0:
        return [0.0] * len(vals)
    out = []
    for v in vals:
        r = float(F32(F32(v) / den))
        out.append(math.copysign(_nearest(abs(r), E2M1_GRID), r) * s * float(g32))
    return out


def scalar_qdq_row(row, g: float):
    out = []
    for b in range(0, len(row), 16):
        out.extend(scalar_qdq_block(row[b:b + 16], g))
    return out


def scalar_qdq_matrix(mat):
    """A weight matrix with its own tensor scale (one per matrix)."""
    g = scalar_tensor_scale([v for row in mat for v in row])
    return [scalar_qdq_row(row, g) for row in mat]


def bf16_nearest(v: float) -> float:
    """Round to the nearest bfloat16 (via float32, ties to even), from the bit patterns."""
    u = struct.unpack("<I", struct.pack("<f", float(F32(v))))[0]
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return struct.unpack("<f", struct.pack("<I", u & 0xFFFFFFFF))[0]


def matvec(m, v):
    return [sum(a * b for a, b in zip(row, v)) for row in m]


def restated_forward(w: lo.OracleWeights, x: np.ndarray, k: int, requant_u=True, h_scale="h", h_bf16=True):
    """The NVFP4 layer per token with Python scalars and loops.  The keyword arguments plant the
    mistakes pin 3 looks for; their defaults are the layer as specified."""
    T = x.shape[0]
    xs = [list(map(float, row)) for row in x]
    wr = w.w_router.tolist()
    wd = w.w_down.tolist()
    hs = [[bf16_nearest(v) if h_bf16 else v for v in matvec(wd, xr)] for xr in xs]
    g_x = scalar_tensor_scale([v for r in xs for v in r])
    g_h = scalar_tensor_scale([v for r in hs for v in r])
    xq = [scalar_qdq_row(r, g_x) for r in xs]
    hq = [scalar_qdq_row(r, g_h if h_scale == "h" else g_x) for r in hs]
    w1q = [scalar_qdq_matrix(w.w1(e).tolist()) for e in range(w.n_experts)]
    w2q = [scalar_qdq_matrix(w.w2(e).tolist()) for e in range(w.n_experts)]
    ws1q = scalar_qdq_matrix(w.ws1.tolist())
    ws2q = scalar_qdq_matrix(w.ws2.tolist())
    wup = w.w_up.tolist()
    req = (lambda u: scalar_qdq_row(u, 1.0)) if requant_u else (lambda u: u)
    y = []
    for t in range(T):
        logits = matvec(wr, xs[t])
        sel = sorted(range(len(logits)), key=lambda e: (-logits[e], e))[:k]
        mx = max(logits[e] for e in sel)
        ex = [math.exp(logits[e] - mx) for e in sel]
        gates = [v / sum(ex) for v in ex]
        z = [0.0] * len(hs[t])
        for g, e in zip(gates, sel):
            u = [max(v, 0.0) ** 2 for v in matvec(w1q[e], hq[t])]
            o = matvec(w2q[e], req(u))
            z = [a + g * b for a, b in zip(z, o)]
        us = [max(v, 0.0) ** 2 for v in matvec(ws1q, xq[t])]
        sh = matvec(ws2q, req(us))
        y.append([a + b for a, b in zip(matvec(wup, z), sh)])
    return np.array(y)


# ------------------------------------------------------------------------------------------------
# layers
# ------------------------------------------------------------------------------------------------
def _bf16(a: np.ndarray) -> np.ndarray:
    return inp.f32_to_bf16_bits(np.asarray(a, np.float32))


def random_layer(seed: int, d=32, l=32, n=4, m=32, ms=32, t=24):
    """A small random bf16 layer with activations whose per-call scales differ (g_x != g_h)."""
    rng = np.random.default_rng(seed)
    norm = lambda *s, std=1.0: rng.standard_normal(s).astype(np.float32) * np.float32(std)
    w = inp.LayerWeights(
        w_router=_bf16(norm(n, d, std=d ** -0.5)), b_router=None,
        w_down=_bf16(norm(l, d, std=3 * d ** -0.5)), w_up=_bf16(norm(d, l, std=l ** -0.5)),
        w1=_bf16(norm(n, m, l, std=l ** -0.5)), w2=_bf16(norm(n, l, m, std=m ** -0.5)),
        ws1=_bf16(norm(ms, d, std=d ** -0.5)), ws2=_bf16(norm(d, ms, std=ms ** -0.5)), dtype="bf16")
    x = lo.lift(_bf16(norm(t, d)), "bf16")
    return lo.OracleWeights(w), x


def representable_layer(seed: int):
    """A layer on which every NVFP4 quantisation of the forward is exact.

    d = 64, l = 32, N = 4, K = 2, m = m_s = 32, T = 4.  x blocks: element 0 is +-6 s g (the block
    amax), elements 1..14 are 0 or +-1 s g, element 15 is 0, with g = 2^-10 and s a power of two in
    1..8; token 0's block 0 has s = 448 and nothing but its amax, which fixes amax(x) = 2688 g, so the
    dynamic tensor scale is exactly g.  h = x[:, :32] (W_down = [I 0]).  Each weight matrix has one
    element 2688 * 4 (tensor scale exactly 4) alone in a row that meets only zeros; every other row
    has one weight +-1.5 * 2^8 (block scale 16, code 6) that picks an element 1..14 of one block, the
    same block for all rows of a 16-row output block, so each u / u_s block holds 0 and one value
    (1.5 * 2^8 * s g)^2, representable with tensor scale 1."""
    rng = np.random.default_rng(seed)
    d, l, n, k, m, ms, t = 64, 32, 4, 2, 32, 32, 4
    g = 2.0 ** -10
    x = np.zeros((t, d))
    for tt in range(t):
        for b in range(d // 16):
            s = 448.0 if (tt == 0 and b == 0) else 2.0 ** rng.integers(0, 4)
            x[tt, 16 * b] = rng.choice([-6.0, 6.0]) * s * g
            if not (tt == 0 and b == 0):
                x[tt, 16 * b + 1:16 * b + 15] = rng.choice([-1.0, 0.0, 1.0], 14) * s * g
    big, c = 2688.0 * 4.0, 1.5 * 2.0 ** 8

    def selector(rows, cols, src_block_of_row_block, dummy_row, dummy_col):
        a = np.zeros((rows, cols))
        for r in range(rows):
            if r == dummy_row:
                a[r, dummy_col] = big
                continue
            blk = src_block_of_row_block[r // 16]
            a[r, 16 * blk + rng.integers(1, 15)] = rng.choice([-c, c])
        return a

    w_down = np.zeros((l, d))
    w_down[np.arange(l), np.arange(l)] = 1.0
    # W1_e rows pick h blocks; the dummy sits at h column 31 (element 15 of block 1: always 0)
    w1 = np.stack([selector(m, l, [0, 1], 3, 31) for _ in range(n)])
    # W2_e rows pick u elements; the dummy row's column 3 is u[3], which is always 0 (dummy row of W1)
    w2 = np.zeros((n, l, m))
    for e in range(n):
        for r in range(l):
            if r == 5:
                w2[e, r, 3] = big
            else:
                col = rng.integers(0, m)
                col = col if col != 3 else 4
                w2[e, r, col] = rng.choice([-c, c])
    ws1 = selector(ms, d, [2, 3], 7, 63)
    ws2 = np.zeros((d, ms))
    for r in range(d):
        if r == 9:
            ws2[r, 7] = big
        else:
            col = rng.integers(0, ms)
            ws2[r, col if col != 7 else 8] = rng.choice([-c, c])
    lw = inp.LayerWeights(w_router=_bf16(rng.standard_normal((n, d)) / 8), b_router=None, w_down=_bf16(w_down),
                          w_up=_bf16(rng.standard_normal((d, l)) / 8), w1=_bf16(w1), w2=_bf16(w2), ws1=_bf16(ws1),
                          ws2=_bf16(ws2), dtype="bf16")
    ow = lo.OracleWeights(lw)
    xb = lo.lift(_bf16(x), "bf16")
    assert np.array_equal(xb, x)                       # every value above is bf16-exact
    return ow, xb, k


# ------------------------------------------------------------------------------------------------
# pins
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_nvfp4_forward_equals_bf16_forward_on_a_representable_layer(seed):
    ow, x, k = representable_layer(seed)
    # the construction really is representable: every quantise-dequantise below is the identity
    g_x = nv.tensor_scale(x.astype(np.float32))
    assert g_x == np.float32(2.0 ** -10)
    assert np.array_equal(nv.qdq(x.astype(np.float32), g_x), x)
    h = x @ ow.w_down.T
    assert np.array_equal(nv.bf16_round(h), h) and nv.tensor_scale(h.astype(np.float32)) == g_x
    for e in range(ow.n_experts):
        for wm in (ow.w1(e), ow.w2(e)):
            assert np.array_equal(nv.qdq(wm.astype(np.float32)), wm)
        u = lo.sqrelu(h @ ow.w1(e).T)
        assert np.array_equal(nv.qdq(u.astype(np.float32), np.float32(1.0)), u) and u.any()
    for wm in (ow.ws1, ow.ws2):
        assert np.array_equal(nv.qdq(wm.astype(np.float32)), wm)
    us = lo.sqrelu(x @ ow.ws1.T)
    assert np.array_equal(nv.qdq(us.astype(np.float32), np.float32(1.0)), us) and us.any()
    # the pin
    a = nv.forward_nvfp4(ow, x, k)
    b = lo.forward(ow, x, k)
    assert np.array_equal(a["idx"], b["idx"])
    assert np.abs(a["y"] - b["y"]).max() <= 1e-12 * np.abs(b["y"]).max()


@pytest.fixture(scope="module")
def rand_layer():
    ow, x = random_layer(11)
    ref = nv.forward_nvfp4(ow, x, 2)
    return ow, x, ref


def test_nvfp4_forward_matches_the_scalar_restatement(rand_layer):
    ow, x, ref = rand_layer
    y = restated_forward(ow, x, 2)
    scale = np.abs(ref["y"]).max()
    assert np.abs(y - ref["y"]).max() <= 1e-12 * scale


@pytest.mark.parametrize("mistake", [{"requant_u": False}, {"h_scale": "x"}, {"h_bf16": False}],
                         ids=["u_not_requantised", "h_with_g_x", "h_not_rounded_to_bf16"])
def test_planted_mistakes_change_the_result(rand_layer, mistake):
    ow, x, ref = rand_layer
    assert nv.tensor_scale(x.astype(np.float32)) != ref["g_h"]   # the layer tells g_x and g_h apart
    y = restated_forward(ow, x, 2, **mistake)
    assert np.abs(y - ref["y"]).max() > 1e-6 * np.abs(ref["y"]).max()
