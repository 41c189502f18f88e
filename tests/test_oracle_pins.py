"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against brute force, a closed form, an invariant of the LatentMoE
definition ("Nemotron 3 Super" notes, section 3.2) or a library routine, chosen so that a dropped
term, a sign error, a transposed operand or a wrong index in the oracle fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest

import lmoe_inputs as inp
from oracle import lmoe_oracle as lo
from oracle import nvfp4 as nv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------------
# helpers: small random layers held directly in float64 (no bf16 rounding needed for pins)
# ------------------------------------------------------------------------------------------------
class _W:
    def __init__(self, rng, d, l, n, m, ms, bias=False):
        self.w_router = rng.standard_normal((n, d))
        self.b_router = rng.standard_normal(n) if bias else None
        self.w_down = rng.standard_normal((l, d)) / math.sqrt(d)
        self.w_up = rng.standard_normal((d, l)) / math.sqrt(l)
        self._w1 = rng.standard_normal((n, m, l)) / math.sqrt(l)
        self._w2 = rng.standard_normal((n, l, m)) / math.sqrt(m)
        self.ws1 = rng.standard_normal((ms, d)) / math.sqrt(d)
        self.ws2 = rng.standard_normal((d, ms)) / math.sqrt(ms)
        self.n_experts = n

    def w1(self, e):
        return self._w1[e]

    def w2(self, e):
        return self._w2[e]


def _python_layer(W, x, k):
    """The layer in plain Python loops (lists and math only), for tiny sizes."""
    T, d = x.shape
    l = W.w_down.shape[0]
    n = W.n_experts
    ys, idxs, gates = [], [], []
    for t in range(T):
        xt = [float(v) for v in x[t]]
        logit = []
        for e in range(n):
            acc = 0.0
            for j in range(d):
                acc += xt[j] * float(W.w_router[e, j])
            if W.b_router is not None:
                acc += float(W.b_router[e])
            logit.append(acc)
        order = sorted(range(n), key=lambda e: (-logit[e], e))[:k]
        mx = max(logit[e] for e in order)
        ex = [math.exp(logit[e] - mx) for e in order]
        g = [v / sum(ex) for v in ex]
        h = [sum(float(W.w_down[i, j]) * xt[j] for j in range(d)) for i in range(l)]
        z = [0.0] * l
        for gk, e in zip(g, order):
            w1, w2 = W.w1(e), W.w2(e)
            u = []
            for a in range(w1.shape[0]):
                v = sum(float(w1[a, i]) * h[i] for i in range(l))
                u.append(max(v, 0.0) ** 2)
            for i in range(l):
                z[i] += gk * sum(float(w2[i, a]) * u[a] for a in range(len(u)))
        us = []
        for a in range(W.ws1.shape[0]):
            v = sum(float(W.ws1[a, j]) * xt[j] for j in range(d))
            us.append(max(v, 0.0) ** 2)
        y = []
        for j in range(d):
            v = sum(float(W.w_up[j, i]) * z[i] for i in range(l))
            v += sum(float(W.ws2[j, a]) * us[a] for a in range(len(us)))
            y.append(v)
        ys.append(y)
        idxs.append(order)
        gates.append(g)
    return np.array(ys), np.array(idxs), np.array(gates)


# ------------------------------------------------------------------------------------------------
# top-K
# ------------------------------------------------------------------------------------------------
def _brute_topk(row, k):
    """Among all k-subsets with the largest logit sum, the lexicographically smallest index tuple;
    returned in (logit desc, index asc) order."""
    best, best_set = None, None
    for sub in itertools.combinations(range(len(row)), k):
        s = sum(row[i] for i in sub)
        if best is None or s > best or (s == best and sub < best_set):
            best, best_set = s, sub
    return sorted(best_set, key=lambda i: (-row[i], i))


@pytest.mark.parametrize("n,k", [(4, 1), (4, 3), (8, 2), (12, 4), (16, 4), (16, 1)])
def test_topk_matches_bruteforce_random(n, k):
    rng = np.random.default_rng(100 + n * 10 + k)
    logits = rng.standard_normal((60, n))
    got = lo.topk(logits, k)
    for r in range(logits.shape[0]):
        assert list(got[r]) == _brute_topk(list(logits[r]), k)


@pytest.mark.parametrize("n,k", [(6, 2), (8, 3), (10, 4)])
def test_topk_matches_bruteforce_with_exact_ties(n, k):
    rng = np.random.default_rng(7 + n)
    logits = rng.integers(-2, 3, size=(80, n)).astype(np.float64)   # many exact ties
    got = lo.topk(logits, k)
    for r in range(logits.shape[0]):
        assert list(got[r]) == _brute_topk(list(logits[r]), k)


def test_topk_hand_cases():
    assert lo.topk(np.array([[1.0, 1.0, 1.0, 0.0]]), 2).tolist() == [[0, 1]]
    assert lo.topk(np.array([[0.0, 2.0, -1.0, 2.0]]), 3).tolist() == [[1, 3, 0]]
    assert lo.topk(np.array([[-5.0, -1.0, -3.0]]), 1).tolist() == [[1]]


# ------------------------------------------------------------------------------------------------
# gates
# ------------------------------------------------------------------------------------------------
def test_gates_sum_to_one_sorted_and_k1():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((100, 32)) * 3
    idx = lo.topk(logits, 6)
    g = lo.softmax_gates(logits, idx)
    assert np.allclose(g.sum(axis=1), 1.0, atol=1e-12, rtol=0)
    assert np.all(np.diff(g, axis=1) <= 0)
    g1 = lo.softmax_gates(logits, lo.topk(logits, 1))
    assert np.all(g1 == 1.0)


def test_gates_closed_form_two_experts():
    # softmax of two logits a > b is the logistic function of a - b
    logits = np.array([[0.3, 1.7, -2.0]])
    idx = lo.topk(logits, 2)
    g = lo.softmax_gates(logits, idx)
    a, b = 1.7, 0.3
    assert idx.tolist() == [[1, 0]]
    assert abs(g[0, 0] - 1.0 / (1.0 + math.exp(b - a))) < 1e-15
    assert abs(g[0, 1] - 1.0 / (1.0 + math.exp(a - b))) < 1e-15


# ------------------------------------------------------------------------------------------------
# whole layer
# ------------------------------------------------------------------------------------------------
def test_layer_matches_python_loops():
    rng = np.random.default_rng(11)
    W = _W(rng, d=6, l=3, n=5, m=4, ms=3, bias=True)
    x = rng.standard_normal((4, 6))
    out = lo.forward(W, x, 2)
    y, idx, g = _python_layer(W, x, 2)
    assert out["idx"].tolist() == idx.tolist()
    assert np.allclose(out["gate"], g, rtol=0, atol=1e-14)
    assert np.allclose(out["y"], y, rtol=1e-12, atol=1e-12)


def test_single_expert_reduces_to_dense_ffn():
    """N = K = 1: the gate is 1 and the layer is the dense FFN W_up W2 sqrelu(W1 W_down x) plus the
    shared expert."""
    rng = np.random.default_rng(12)
    W = _W(rng, d=8, l=4, n=1, m=6, ms=5)
    x = rng.standard_normal((7, 8))
    out = lo.forward(W, x, 1)
    dense = np.maximum((x @ W.w_down.T) @ W.w1(0).T, 0) ** 2 @ W.w2(0).T @ W.w_up.T
    dense += np.maximum(x @ W.ws1.T, 0) ** 2 @ W.ws2.T
    assert np.all(out["gate"] == 1.0)
    assert np.allclose(out["y"], dense, rtol=1e-12, atol=1e-12)


def test_single_expert_degree_two_homogeneity():
    """With N = K = 1 every path is a squared ReLU between linear maps: y(a x) = a^2 y(x), a > 0."""
    rng = np.random.default_rng(13)
    W = _W(rng, d=8, l=4, n=1, m=6, ms=5)
    x = rng.standard_normal((5, 8))
    y1 = lo.forward(W, x, 1)["y"]
    y2 = lo.forward(W, 2.5 * x, 1)["y"]
    assert np.allclose(y2, 6.25 * y1, rtol=1e-12, atol=1e-12)


def test_identity_projections_equal_standard_moe():
    """l = d with W_down = W_up = I is a standard MoE: y = sum_k g_k W2 sqrelu(W1 x) + shared."""
    rng = np.random.default_rng(14)
    d, n, k = 6, 7, 3
    W = _W(rng, d=d, l=d, n=n, m=5, ms=4)
    W.w_down = np.eye(d)
    W.w_up = np.eye(d)
    x = rng.standard_normal((9, d))
    out = lo.forward(W, x, k)
    for t in range(x.shape[0]):
        logit = W.w_router @ x[t]
        sel = sorted(range(n), key=lambda e: (-logit[e], e))[:k]
        w = np.exp(logit[sel] - logit[sel].max())
        w /= w.sum()
        ref = sum(w[i] * (W.w2(e) @ (np.maximum(W.w1(e) @ x[t], 0) ** 2)) for i, e in enumerate(sel))
        ref = ref + W.ws2 @ (np.maximum(W.ws1 @ x[t], 0) ** 2)
        assert np.allclose(out["y"][t], ref, rtol=1e-12, atol=1e-12)


def test_standard_moe_without_projections():
    """A layer given without W_down / W_up (zero-row arrays) runs its experts on x: it equals the
    per-token loop of the standard MoE and the l = d layer with identity projections."""
    rng = np.random.default_rng(15)
    d, n, k = 6, 7, 3
    W = _W(rng, d=d, l=d, n=n, m=5, ms=4)
    x = rng.standard_normal((9, d))
    W.w_down, W.w_up = np.eye(d), np.eye(d)
    ident = lo.forward(W, x, k)["y"]
    W.w_down, W.w_up = np.zeros((0, d)), np.zeros((d, 0))
    out = lo.forward(W, x, k)
    assert np.allclose(out["y"], ident, rtol=1e-13, atol=1e-13)
    for t in range(x.shape[0]):
        logit = W.w_router @ x[t]
        sel = sorted(range(n), key=lambda e: (-logit[e], e))[:k]
        w = np.exp(logit[sel] - logit[sel].max())
        w /= w.sum()
        ref = sum(w[i] * (W.w2(e) @ (np.maximum(W.w1(e) @ x[t], 0) ** 2)) for i, e in enumerate(sel))
        ref = ref + W.ws2 @ (np.maximum(W.ws1 @ x[t], 0) ** 2)
        assert np.allclose(out["y"][t], ref, rtol=1e-12, atol=1e-12)


def test_standard_budget_matches_the_latent_layer():
    """N = N' l / d and K = K' l / d (rounded up): the standard layer holds the Super layer's
    expert parameters and about its active expert weights per token."""
    sup, std = inp.SUPER, inp.STANDARD
    assert std.n_experts == sup.n_experts * sup.latent // sup.d
    assert std.top_k == math.ceil(sup.top_k * sup.latent / sup.d)
    e_sup = sup.n_experts * 2 * sup.expert_ffn * sup.latent
    e_std = std.n_experts * 2 * std.expert_ffn * std.d
    assert e_sup == e_std
    act_sup = sup.top_k * 2 * sup.expert_ffn * sup.latent + 2 * sup.latent * sup.d
    act_std = std.top_k * 2 * std.expert_ffn * std.d
    assert abs(act_std / act_sup - 1) < 0.1


def test_latent_sum_equals_sum_of_up_projections():
    """W_up is linear: up-projecting the latent sum equals summing the up-projected expert outputs."""
    rng = np.random.default_rng(15)
    W = _W(rng, d=10, l=4, n=6, m=5, ms=3)
    x = rng.standard_normal((8, 10))
    out = lo.forward(W, x, 3)
    shared = np.maximum(x @ W.ws1.T, 0) ** 2 @ W.ws2.T
    h = x @ W.w_down.T
    for t in range(x.shape[0]):
        acc = np.zeros(10)
        for kk in range(3):
            e = out["idx"][t, kk]
            o = W.w2(e) @ (np.maximum(W.w1(e) @ h[t], 0) ** 2)
            acc += W.w_up @ (out["gate"][t, kk] * o)
        assert np.allclose(out["y"][t] - shared[t], acc, rtol=1e-12, atol=1e-12)


def test_token_permutation_equivariance():
    rng = np.random.default_rng(16)
    W = _W(rng, d=8, l=4, n=6, m=5, ms=3)
    x = rng.standard_normal((11, 8))
    p = rng.permutation(11)
    a = lo.forward(W, x, 2)
    b = lo.forward(W, x[p], 2)
    assert np.array_equal(a["idx"][p], b["idx"])
    assert np.allclose(a["y"][p], b["y"], rtol=1e-13, atol=1e-13)


def test_expert_relabelling_invariance():
    rng = np.random.default_rng(17)
    W = _W(rng, d=8, l=4, n=6, m=5, ms=3, bias=True)
    x = rng.standard_normal((10, 8))
    a = lo.forward(W, x, 3)
    perm = rng.permutation(6)          # new expert j is old expert perm[j]
    W2 = _W(rng, d=8, l=4, n=6, m=5, ms=3)
    W2.w_router = W.w_router[perm]
    W2.b_router = W.b_router[perm]
    W2.w_down, W2.w_up, W2.ws1, W2.ws2 = W.w_down, W.w_up, W.ws1, W.ws2
    W2._w1 = W._w1[perm]
    W2._w2 = W._w2[perm]
    b = lo.forward(W2, x, 3)
    assert np.allclose(a["y"], b["y"], rtol=1e-13, atol=1e-13)
    assert np.array_equal(perm[b["idx"]], a["idx"])


# ------------------------------------------------------------------------------------------------
# dispatch (integer grouping)
# ------------------------------------------------------------------------------------------------
def test_dispatch_bruteforce():
    rng = np.random.default_rng(18)
    n, k, t = 9, 3, 40
    idx = np.stack([rng.permutation(n)[:k] for _ in range(t)]).astype(np.int32)
    counts, offsets, row_of, tok_of_row = lo.dispatch(idx, n)
    # brute force: walk assignments in (t, k) order, appending to per-expert lists
    lists = [[] for _ in range(n)]
    for tt in range(t):
        for kk in range(k):
            lists[idx[tt, kk]].append((tt, kk))
    rows = {}
    r = 0
    for e in range(n):
        assert counts[e] == len(lists[e]) and offsets[e] == r
        for (tt, kk) in lists[e]:
            rows[(tt, kk)] = r
            r += 1
    assert offsets[n] == t * k
    for (tt, kk), rr in rows.items():
        assert row_of[tt, kk] == rr and tok_of_row[rr] == tt


# ------------------------------------------------------------------------------------------------
# near ties
# ------------------------------------------------------------------------------------------------
def test_near_tie_detection():
    l = np.array([[3.0, 2.0, 1.0, 0.0],
                  [3.0, 2.0, 2.0 - 1e-6, 0.0],     # K-th vs (K+1)-th within eps (K=2)
                  [3.0, 3.0 - 5e-6, 1.0, 0.0],     # order among selected within eps
                  [3.0, 2.0, 2.0 - 1e-4, 0.0]])
    m = lo.near_tie_tokens(l, 2, 1e-5)
    assert m.tolist() == [False, True, True, False]


# ------------------------------------------------------------------------------------------------
# NVFP4
# ------------------------------------------------------------------------------------------------
def _golden_formats():
    e2m1, e4m3 = {}, {}
    with open(os.path.join(GOLDEN, "nvfp4_format.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            kind, code, val = line.split()
            (e2m1 if kind == "e2m1" else e4m3)[int(code, 16)] = float(val)
    return e2m1, e4m3


def test_e2m1_and_e4m3_decode_match_format_table():
    e2m1, e4m3 = _golden_formats()
    for c, v in e2m1.items():
        got = float(nv.e2m1_decode(np.array([c], np.uint8))[0])
        assert got == v and math.copysign(1, got) == math.copysign(1, v)
    for b, v in e4m3.items():
        assert float(nv.e4m3_decode(np.array([b], np.uint8))[0]) == v


def test_e2m1_encode_against_ml_dtypes():
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(19)
    r = np.concatenate([rng.uniform(-7, 7, 20000).astype(np.float32),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, 6.0, 6.5,
                                  0.0, -0.0, 1e-9, -1e-9], np.float32)])
    mine = nv.e2m1_decode(nv.e2m1_encode(r))
    ref = r.astype(ml.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(mine, ref)
    assert np.array_equal(np.signbit(mine), np.signbit(ref))


def test_e4m3_encode_against_ml_dtypes():
    ml = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(20)
    s = np.concatenate([np.exp(rng.uniform(np.log(1e-4), np.log(448), 30000)).astype(np.float32),
                        np.array([0.0, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -6, 448.0, 0.5, 1.0625],
                                 np.float32)])
    mine = nv.e4m3_decode(nv.e4m3_encode(s))
    ref = s.astype(ml.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(mine, ref)
    # every finite non-negative byte round-trips
    b = np.arange(0x7F, dtype=np.uint8)
    assert np.array_equal(nv.e4m3_encode(nv.e4m3_decode(b).astype(np.float32)), b)
    # saturation
    assert nv.e4m3_decode(nv.e4m3_encode(np.array([470.0, 1e6], np.float32))).tolist() == [448.0, 448.0]


@pytest.mark.parametrize("scale_byte", [0x01, 0x38, 0x7E, 0x2B])
def test_hand_built_blocks_round_trip_exactly(scale_byte):
    """A block built from any 16 E2M1 codes (one of them +-6) and an E4M3 scale s, with g = 1,
    is quantised back to exactly those codes and that scale, and dequantises to code * s."""
    _, e4m3 = _golden_formats()
    s = float(nv.e4m3_decode(np.array([scale_byte], np.uint8))[0])
    codes = np.array([[7, 1, 2, 3, 4, 5, 6, 0, 9, 10, 11, 12, 13, 14, 15, 8],
                      [15, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 1]], np.uint8)
    vals = (nv.e2m1_decode(codes) * s).astype(np.float32)
    c, sb, g = nv.quantize(vals, np.float32(1.0))
    assert np.array_equal(sb[:, 0], [scale_byte, scale_byte])
    # +0 and -0 both dequantise to zero; compare values and the sign of non-zeros
    assert np.array_equal(nv.e2m1_decode(c), nv.e2m1_decode(codes))
    assert np.array_equal(nv.dequantize(c, sb, g), nv.e2m1_decode(codes) * s)


def test_rne_ties_and_saturation():
    # block amax 6 with g = 1 gives s = 1 exactly; the other elements hit each rounding midpoint
    v = np.array([[6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, 0, 0, 0, 0, 0, 0]], np.float32)
    c, sb, g = nv.quantize(v, np.float32(1.0))
    assert sb[0, 0] == 0x38
    assert nv.dequantize(c, sb, g)[0, :10].tolist() == [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -0.0, -4.0]
    # amax 6.375 -> s = 1.0625 rounds (tie) to 1.0 in E4M3; the amax element then saturates at 6
    v2 = np.zeros((1, 16), np.float32)
    v2[0, 0] = 6.375
    v2[0, 1] = -3.0
    c2, sb2, _ = nv.quantize(v2, np.float32(1.0))
    assert sb2[0, 0] == 0x38 and nv.e2m1_decode(c2)[0, :2].tolist() == [6.0, -3.0]


def test_oracle_bf16_round_against_ml_dtypes():
    ml = pytest.importorskip("ml_dtypes")
    r = np.concatenate([np.random.default_rng(24).standard_normal(20000) * 7,
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 1e-30]])
    ref = r.astype(np.float32).astype(ml.bfloat16).astype(np.float64)
    assert np.array_equal(nv.bf16_round(r), ref)


def test_zero_block_and_zero_tensor():
    v = np.zeros((2, 32), np.float32)
    v[1, 16:] = np.linspace(-1, 1, 16)
    c, sb, g = nv.quantize(v)
    assert np.all(sb[0] == 0) and sb[1, 0] == 0 and np.all(nv.e2m1_decode(c[:, :16]) == 0)
    assert nv.tensor_scale(np.zeros((3, 16), np.float32)) == 1.0


def test_per_tensor_scale_puts_tensor_amax_at_448_times_6():
    rng = np.random.default_rng(21)
    a = rng.standard_normal((8, 64)).astype(np.float32)
    c, sb, g = nv.quantize(a)
    amax = np.max(np.abs(a))
    assert g == np.float32(amax / np.float32(2688.0))
    # the block holding the tensor amax gets the largest scale (448, up to one fp32 rounding)
    r, col = np.unravel_index(np.argmax(np.abs(a)), a.shape)
    assert nv.e4m3_decode(sb[r, col // 16:col // 16 + 1])[0] == 448.0


def test_qdq_idempotent_and_error_bound():
    rng = np.random.default_rng(22)
    a = rng.standard_normal((16, 128)).astype(np.float32)
    q1 = nv.qdq(a)
    c, sb, g = nv.quantize(a)
    q2 = nv.qdq(q1.astype(np.float32), g)
    assert np.array_equal(q1, q2)
    # relative error per element is bounded by half an E2M1 step (<= 1/4 of the block scale unit
    # at the top binade) plus the E4M3 scale rounding; loosely: |err| <= 0.5 * s * g * 2 per block
    s = nv.e4m3_decode(sb).astype(np.float64) * float(g)
    err = np.abs(q1 - a).reshape(16, 8, 16)
    assert np.all(err <= s[..., None] * 1.0 + 1e-12)


# ------------------------------------------------------------------------------------------------
# per-block MSE weight scales
# ------------------------------------------------------------------------------------------------
_E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e4m3_value(code):
    """E4M3 value from its bit fields (bias 7; exponent field 0 is subnormal), written out here."""
    e, m = code >> 3, code & 7
    return m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)


def _e2m1_round(r):
    """Nearest E2M1 magnitude to |r| (ties to the even index, above 6 saturates), by scanning."""
    a = min(abs(r), 6.0)
    best = None
    for i, gv in enumerate(_E2M1_GRID):
        dist = abs(a - gv)
        if best is None or dist < best[0] or (dist == best[0] and i % 2 == 0):
            best = (dist, i, gv)
    return math.copysign(best[2], r)


def _bruteforce_choice(blk, g):
    """Scale code with the smallest float64 squared error over the window c0+1, c0, c0-1..c0-6,
    plus every candidate's error (quotients v / (s*g) taken in float32 as the method defines)."""
    g32 = np.float32(g)
    c0 = int(nv.e4m3_encode(np.array([np.float32(np.max(np.abs(blk)) / np.float32(6 * g32))]))[0])
    errs = {}
    for c in range(max(c0 - 6, 1 if c0 > 0 else 0), min(c0 + 1, 0x7E) + 1):
        s = _e4m3_value(c)
        den = np.float32(np.float32(s) * g32)
        q = [_e2m1_round(float(np.float32(np.float32(v) / den))) if den > 0 else 0.0 for v in blk]
        errs[c] = sum((float(v) - qi * s * float(g32)) ** 2 for v, qi in zip(blk, q))
    return min(errs, key=lambda c: (errs[c], c != c0)), errs


def test_mse_choice_matches_bruteforce_argmin():
    rng = np.random.default_rng(31)
    # heavy tails make clipping the block's largest element worthwhile in some blocks
    a = (rng.standard_t(3, size=(24, 256)) * 0.02).astype(np.float32)
    g = nv.tensor_scale(a)
    _, sb, _ = nv.quantize_mse(a, g)
    blk = a.reshape(24, 16, 16)
    changed = close = 0
    for r in range(24):
        for b in range(16):
            c, errs = _bruteforce_choice(blk[r, b], g)
            got = int(sb[r, b])
            if got != c:
                # only where the float32 and float64 error sums order two candidates differently
                assert abs(errs[got] - errs[c]) <= 1e-5 * max(errs[c], 1e-30), (r, b, got, c, errs)
                close += 1
            changed += got != nv.quantize(blk[r, b][None, :], g)[1][0, 0]
    assert changed > 0 and close <= 2


def test_mse_hand_block_prefers_a_smaller_scale():
    # g = 1.  Squared block errors by hand: s = 1.125: 0.5625 + 15 * 0.015625 = 0.796875;
    # s = 1 (the amax rule; the fifteen 1.25 ties round to 1): 15 * 0.0625 = 0.9375;
    # s = 0.9375: 6 saturates to 5.625 and 1.25 / 0.9375 = 1.33 goes to 1.5 (1.40625):
    #   0.140625 + 15 * 0.0244140625 = 0.5068359375;  s = 0.875: 0.5625 + 15 * 0.00390625 = 0.62109375;
    # smaller scales clip the 6 harder.
    blk = np.array([[6.0] + [1.25] * 15], np.float32)
    c_amax = int(nv.quantize(blk, np.float32(1))[1][0, 0])
    codes, sb, _ = nv.quantize_mse(blk, np.float32(1))
    assert _e4m3_value(c_amax) == 1.0 and _e4m3_value(int(sb[0, 0])) == 0.9375
    deq = nv.dequantize(codes, sb, np.float32(1))
    assert ((deq - blk) ** 2).sum() == 0.5068359375


def test_mse_keeps_exactly_representable_blocks():
    rng = np.random.default_rng(32)
    g = np.float32(2.0 ** -7)                           # a power of two keeps q * s * g exact
    for code in (0x08, 0x30, 0x38, 0x50, 0x7E):
        s = _e4m3_value(code)
        vals = rng.choice(_E2M1_GRID, size=16) * rng.choice([-1.0, 1.0], size=16)
        vals[0] = 6.0                                   # the block amax pins the amax scale to s
        blk = (vals * s * float(g)).astype(np.float32)[None, :]
        codes, sb, _ = nv.quantize_mse(blk, g)
        assert int(sb[0, 0]) == int(nv.quantize(blk, g)[1][0, 0])
        assert np.array_equal(nv.dequantize(codes, sb, g), blk.astype(np.float64))


def test_mse_candidate_window_edges():
    assert nv.mse_candidates(0x38) == [0x38, 0x39, 0x37, 0x36, 0x35, 0x34, 0x33, 0x32]
    assert nv.mse_candidates(0x7E) == [0x7E, 0x7D, 0x7C, 0x7B, 0x7A, 0x79, 0x78]
    assert nv.mse_candidates(3) == [3, 4, 2, 1]
    assert nv.mse_candidates(0) == [0, 1]


def test_mse_never_worse_than_amax_and_lower_on_average():
    rng = np.random.default_rng(33)
    a = (rng.standard_normal((64, 512)) / math.sqrt(512)).astype(np.float32)
    g = nv.tensor_scale(a)
    c0, s0, _ = nv.quantize(a, g)
    c1, s1, _ = nv.quantize_mse(a, g)
    e0 = ((nv.dequantize(c0, s0, g) - a) ** 2).reshape(64, 32, 16).sum(-1)
    e1 = ((nv.dequantize(c1, s1, g) - a) ** 2).reshape(64, 32, 16).sum(-1)
    assert np.all(e1 <= e0 * (1 + 1e-6) + 1e-30)
    assert e1.sum() < 0.9 * e0.sum()


# ------------------------------------------------------------------------------------------------
# shapes and workloads
# ------------------------------------------------------------------------------------------------
def test_super_shape_matches_architecture_table():
    vals = {}
    with open(os.path.join(GOLDEN, "super_layer_shape.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split()
            vals[k] = int(v)
    s = inp.SUPER
    assert (s.d, s.expert_ffn, s.shared_ffn, s.n_experts, s.top_k, s.latent) == (
        vals["model_dim"], vals["expert_hidden"], vals["shared_expert_hidden"],
        vals["experts_per_layer"], vals["top_k"], vals["moe_latent_dim"])


def test_ultra_shape_matches_the_ultra_summary():
    vals = {}
    with open(os.path.join(GOLDEN, "ultra_layer_shape.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split()
            vals[k] = int(v)
    u = inp.ULTRA
    assert (u.n_experts, u.top_k, u.expert_ffn, u.shared_ffn) == (
        vals["experts_per_layer"], vals["top_k"], vals["expert_hidden"], vals["shared_expert_hidden"])
    # not on that page: Super's model and latent dimensions are kept
    assert (u.d, u.latent) == (inp.SUPER.d, inp.SUPER.latent)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], np.float32)
    b = inp.bf16_bits_to_f32(inp.f32_to_bf16_bits(x))
    assert b.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5]
    ml = pytest.importorskip("ml_dtypes")
    r = np.random.default_rng(23).standard_normal(10000).astype(np.float32)
    assert np.array_equal(inp.bf16_bits_to_f32(inp.f32_to_bf16_bits(r)),
                          r.astype(ml.bfloat16).astype(np.float32))


def test_skewed_workload_load_profile():
    """The stored router bias gives >= 32 idle experts and a hot expert above 10 % of the tokens."""
    wl = inp.workload("skewed")
    x = lo.lift(inp.make_x(wl), "bf16")
    logits = lo.router_logits(x, lo.lift(inp.make_router(wl), "bf16"),
                              inp.skewed_router_bias().astype(np.float64))
    counts = np.bincount(lo.topk(logits, wl.shape.top_k).ravel(), minlength=wl.shape.n_experts)
    assert (counts == 0).sum() >= 32
    assert counts.max() > 0.10 * wl.tokens
    assert counts.sum() == wl.tokens * wl.shape.top_k
    # Zipf-like: the sorted non-zero loads fall with rank, the tail is at least 10x below the head
    srt = np.sort(counts)[::-1]
    assert srt[100] < srt[0] and srt[400] * 10 < srt[0]
