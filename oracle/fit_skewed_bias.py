"""Fit the per-expert router bias of the skewed workload and store it as input data.

Run once, offline:  python -m oracle.fit_skewed_bias
Writes lmoe_inputs/skewed_router_bias_f32.txt (512 float32 values as hex bit patterns).

Target.  Each token selects an expert at most once, so one expert can hold at most T of the
T*K assignments (1/K = 4.5 %).  The skewed workload therefore reads "one hot expert with >10 %"
as ">10 % of tokens", and shapes the per-expert token loads as a capped Zipf(s = 1.2) profile:
    L_r = min(T, c * r^-1.2),  r = 1..480 (rank),  L_r = 0 for the last 32 ranks,
with c chosen so that sum_r L_r = T*K.  Ranks map to expert ids through a seeded permutation.

Fit.  Starting from b = 0, 200 rounds of  b_e <- b_e + 0.5 * (ln(L_e + 0.5) - ln(obs_e + 0.5)),
where obs_e is the load of the oracle's own top-K under the current bias; the 32 idle experts get
b = -30 (never selected).  The stored float32 b is what defines the workload: its achieved loads
(recounted from the stored values) are what the tests report.
"""
from __future__ import annotations

import os

import numpy as np

import lmoe_inputs as inp
from . import lmoe_oracle as lo

N_IDLE = 32
ZIPF_S = 1.2
ROUNDS = 200
PERM_SEED = 5


def target_loads(n: int, t: int, k: int) -> np.ndarray:
    ranks = np.arange(1, n - N_IDLE + 1, dtype=np.float64)
    lo_c, hi_c = 1.0, float(t * k) * 10
    for _ in range(200):                      # bisection on c
        c = 0.5 * (lo_c + hi_c)
        tot = np.minimum(t, c * ranks ** -ZIPF_S).sum()
        lo_c, hi_c = (c, hi_c) if tot < t * k else (lo_c, c)
    loads = np.minimum(t, c * ranks ** -ZIPF_S)
    return np.concatenate([loads, np.zeros(N_IDLE)])


def main() -> None:
    wl = inp.workload("skewed")
    s = wl.shape
    x = lo.lift(inp.make_x(wl), "bf16")
    base = lo.router_logits(x, lo.lift(inp.make_router(wl), "bf16"))
    perm = np.random.Generator(np.random.PCG64(PERM_SEED)).permutation(s.n_experts)
    target = np.empty(s.n_experts)
    target[perm] = target_loads(s.n_experts, wl.tokens, s.top_k)
    idle = target == 0
    b = np.zeros(s.n_experts)
    b[idle] = -30.0
    for _ in range(ROUNDS):
        idx = lo.topk(base + b[None, :], s.top_k)
        obs = np.bincount(idx.ravel(), minlength=s.n_experts)
        upd = 0.5 * (np.log(target + 0.5) - np.log(obs + 0.5))
        b[~idle] += upd[~idle]
    b32 = b.astype(np.float32)
    out = os.path.join(os.path.dirname(inp.__file__), "skewed_router_bias_f32.txt")
    with open(out, "w") as fh:
        fh.write("# router bias of the skewed workload, float32 bit patterns (hex), expert 0..511;"
                 " written by oracle/fit_skewed_bias.py\n")
        bits = b32.view(np.uint32)
        for i in range(0, bits.size, 8):
            fh.write(" ".join(f"{v:08x}" for v in bits[i:i + 8]) + "\n")
    idx = lo.topk(base + b32.astype(np.float64)[None, :], s.top_k)
    obs = np.bincount(idx.ravel(), minlength=s.n_experts)
    print("zero-load experts:", int((obs == 0).sum()), " max load:", int(obs.max()),
          f"({obs.max() / wl.tokens:.1%} of tokens)", " sum:", int(obs.sum()))


if __name__ == "__main__":
    main()
