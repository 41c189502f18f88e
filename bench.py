"""Throughput of the B200 LatentMoE layer (Super shape) on seeded synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--no-cpu-baseline] [--no-prefill]

Workloads (lmoe_inputs): decode (default), prefill, skewed, tiny, decode_nvfp4, prefill_nvfp4, the
Ultra-width and standard-MoE variants, and the small profiling cases.

One step = one full forward of the layer (router, top-K, dispatch, W_down, routed experts, combine,
W_up, shared expert) over one batch.  The default workload is the Super-shaped decode/verify batch
(T = 256); the same run then also times the T = 16384 prefill batch on the same layer and reports it
as the line's "prefill" object (its own steps, roofline, e2e and cpu_baseline), so one line carries
both halves of the metric.  With N > 1 (torchrun, one process per GPU) every rank runs an
independent replica: the layer has no cross-GPU step, so nothing is exchanged and scaling is weak.

Prints ONE JSON line on rank 0.  `value` is whole-job tokens/s with inputs resident in HBM; `e2e`
is the same through lmoe_forward_host (pinned host x in, y/idx/gate out, copies inside the timed
region); `roofline` reports the dominant kernel's algorithmic bytes (or FLOPs) per launch over its
CUDA-event duration against the measured peak, from a second, identical timed loop that records the
library's per-stage events (`profiled_ms_per_step`; the headline loop runs without them);
`cpu_baseline` times the fp64 oracle on a bounded sample on the host cores.  `--impl reference`
times that oracle alone as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import lmoe_inputs as inp  # noqa: E402

METRIC = "LatentMoE layer tokens/s (Super shape, T=256 & 16K); % of HBM / TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_STEPS = {"tiny": 200, "decode": 400, "skewed": 40, "prefill": 20}
DEFAULT_STEPS.update({"decode_small": 400, "decode_nvfp4": 400, "prefill_nvfp4": 20, "nvfp4_tiny": 200,
                      "nvfp4_mid": 100, "ultra_decode": 200, "ultra_decode_nvfp4": 200, "ultra_prefill": 10,
                      "standard_decode": 400, "standard_prefill": 20, "prefill_small": 20})


# DRAM traffic per launch of the expert GEMMs over their algorithmic bytes (dram__bytes_read.sum +
# dram__bytes_write.sum from ncu section captures, summarised under profiles/): the decode NVFP4
# capture is the full workload; the others are smaller cases of the same regime (Super dims with
# 128 experts: T = 64 for decode, T = 4096 for bf16 and NVFP4 prefill), scaled to a launch by its algorithmic
# bytes, which grow with the units processed.  The prefill ratios hold where the library runs the
# same GEMM variants as the capture (expert up on one CTA: at least one full 256-token tile per
# expert on average; expert down as CTA pairs).  Valid only while the GEMM's sources are the ones
# captured (TRAFFIC_SOURCES_SHA256); otherwise the roofline reports no traffic.
TRAFFIC_RATIO = {
    ("bf16", "decode", "expert_up"): 0.998, ("bf16", "decode", "expert_down"): 1.001,
    ("nvfp4", "decode", "expert_up"): 1.384, ("nvfp4", "decode", "expert_down"): 1.494,
    ("bf16", "prefill", "expert_up"): 0.982, ("bf16", "prefill", "expert_down"): 1.051,
    ("nvfp4", "prefill", "expert_up"): 1.457, ("nvfp4", "prefill", "expert_down"): 1.246,
}
TRAFFIC_SOURCES = ("gemm_tc.cuh", "ptx.cuh", "nvfp4.cuh", "lmoe.cu")
TRAFFIC_SOURCES_SHA256 = "5aeb9bc3143e270f9362e872b6c4cf2a8d1ca6985c385975e30c8f2bc0ccc353"


def gemm_sources_sha256() -> str:
    """SHA-256 of the GEMM's code: the sources with comments removed and whitespace runs collapsed, so
    that editing a comment does not invalidate a capture (string literals are kept as they are)."""
    import hashlib
    import re
    token = re.compile(r'"(?:\\.|[^"\\])*"|//[^\n]*|/\*.*?\*/', re.S)
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "latentmoe_expert_layer_b200", "csrc", f)) as fh:
            src = fh.read()
        code = token.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", src)
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------ helpers
def algorithmic_work(wl, counts: np.ndarray):
    """Bytes and FLOPs one forward must move / compute, from the actual routing (counts per expert).

    bf16 weights: 2 bytes per element.  NVFP4 weights and activations: 0.5 byte per element plus one
    E4M3 scale byte per 16 elements (router, W_down and W_up stay bf16 in the NVFP4 variant)."""
    s = wl.shape
    d, l, n, k, m, ms = s.d, s.latent, s.n_experts, s.top_k, s.expert_ffn, s.shared_ffn
    le = s.expert_in        # the experts' input width: l, or d for a standard MoE (l = 0)
    t = wl.tokens
    tk = t * k
    touched = int((counts > 0).sum())
    fp4 = wl.precision == "nvfp4"
    eb = (lambda elems: elems * 0.5 + elems / 16) if fp4 else (lambda elems: elems * 2)
    w_exp = touched * eb(m * le)                    # one expert matrix set (W1 or W2) of the touched experts
    up = {"bytes": w_exp + eb(tk * le) + eb(tk * m), "flops": 2 * tk * m * le}
    down = {"bytes": w_exp + eb(tk * m) + tk * le * 2 + tk * 4, "flops": 2 * tk * m * le}
    # At decode sizes the library folds the shared expert into the two expert launches (its first
    # matrix into the up launch, its second, writing fp32 y_s, into the down launch); their bytes
    # and FLOPs are then part of those launches.  Same condition as the library's split path.
    folded = tk <= 48 * n and (fp4 or t <= 512)
    if folded:
        up["bytes"] += eb(ms * d) + eb(t * d) + eb(t * ms)
        up["flops"] += 2 * t * ms * d
        down["bytes"] += eb(d * ms) + eb(t * ms) + t * d * 4
        down["flops"] += 2 * t * d * ms
    layer_bytes = (2 * w_exp + (n + l) * d * 2 + eb(ms * d) + eb(d * ms) + d * l * 2 + 2 * t * d * 2 + tk * 8)
    layer_flops = 2 * t * ((n + l) * d + ms * d + d * (l + ms)) + 4 * tk * m * le
    return {"expert_up": up, "expert_down": down, "layer": {"bytes": int(layer_bytes), "flops": layer_flops},
            "touched_experts": touched, "expert_weight_bytes": int(2 * w_exp)}


def make_device_layer(wl, device, max_tokens=None):
    import torch

    import latentmoe_expert_layer_b200 as lm
    w = inp.make_weights(wl)
    to = lambda a: (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
                    if w.dtype == "bf16" else torch.from_numpy(np.ascontiguousarray(a))).to(device)
    dev = {k: to(getattr(w, k)) for k in ("w_router", "w_down", "w_up", "w1", "w2", "ws1", "ws2")}
    if wl.shape.latent == 0:          # a standard MoE has no projections
        dev["w_down"] = dev["w_up"] = None
    b = torch.from_numpy(w.b_router).to(device) if w.b_router is not None else None
    layer = lm.LatentMoE(wl.shape, max_tokens or wl.tokens, precision=wl.precision, router_bias=wl.router_bias,
                         device=device.index)
    layer.load_weights(b_router=b, **dev)
    torch.cuda.synchronize(device)
    del dev
    torch.cuda.empty_cache()
    return layer, w


def _oracle_forward(wl):
    from oracle import lmoe_oracle as lo
    from oracle import nvfp4 as nv
    return nv.forward_nvfp4 if wl.precision == "nvfp4" else lo.forward


def cpu_baseline(wl, w, budget_s: float = 20.0):
    """The fp64 oracle, as it stands, on a bounded token sample of the same workload."""
    from oracle import lmoe_oracle as lo
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    ow = lo.OracleWeights(w)
    x = lo.lift(inp.make_x(wl), "bf16")
    fwd = _oracle_forward(wl)
    done, t0, sample = 0, time.perf_counter(), 0
    while time.perf_counter() - t0 < budget_s and done < wl.tokens:
        n = min(4, wl.tokens - done)
        fwd(ow, x[done:done + n], wl.shape.top_k)
        done += n
    el = time.perf_counter() - t0
    return {"value": done / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {done} of the {wl.tokens} tokens, fp64 numpy oracle, {el:.1f} s"}


# ------------------------------------------------------------------------------------------ ranks
def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of every rank's `value` (a device-timed duration): the job's time is its slowest
    replica's.  Every rank calls this at the same point; one all-reduce, none at world == 1."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens: int, steps: int, ms: float) -> float:
    """Tokens every replica processed in `steps` steps of `tokens` tokens, over the max-over-ranks
    time `ms`."""
    return world * tokens * steps / (ms * 1e-3)


# ------------------------------------------------------------------------------------------ arms
def run_reference(args, wl, rank):
    if rank != 0:
        return
    from oracle import lmoe_oracle as lo
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    w = inp.make_weights(wl)
    ow = lo.OracleWeights(w)
    x = lo.lift(inp.make_x(wl), "bf16")
    per_step = 1 if wl.shape.n_experts > 64 else wl.tokens   # bounded sample per step
    pos = 0

    fwd = _oracle_forward(wl)

    def step():
        nonlocal pos
        fwd(ow, x[pos:pos + per_step], wl.shape.top_k)
        pos = (pos + per_step) % max(1, wl.tokens - per_step + 1)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    val = per_step * args.steps / el
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "tokens": wl.tokens, "sample_tokens_per_step": per_step},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{per_step} token(s) of the {wl.tokens}-token batch per step"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def load_stats(counts: np.ndarray, tokens: int) -> dict:
    """Per-expert load of one forward, from the assignment count of every expert."""
    c = np.asarray(counts, np.float64)
    return {"max_over_mean": float(c.max() / max(c.mean(), 1e-30)), "zero_load_experts": int((c == 0).sum()),
            "hottest_share_of_tokens": float(c.max() / tokens), "touched_experts": int((c > 0).sum())}


def measure(layer, w, wl, steps, warmup, world, device, with_cpu_baseline):
    """Time `steps` forwards of workload wl on the loaded layer (after `warmup` untimed ones) and
    return its line's fields: the headline loop without stage events, a second identical loop with
    the library's per-stage events (stage breakdown, dominant kernel), and the end-to-end loop
    through lmoe_forward_host.  Durations are device-timed and taken as the max over ranks."""
    import torch
    import torch.distributed as dist

    x_bits = inp.make_x(wl)
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(device)
    t = wl.tokens
    y = torch.empty((t, wl.shape.d), dtype=torch.bfloat16, device=device)
    idx = torch.empty((t, wl.shape.top_k), dtype=torch.int32, device=device)
    gate = torch.empty((t, wl.shape.top_k), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(warmup):
        layer.forward(x, y, idx, gate)
    torch.cuda.synchronize(device)
    st = layer.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    counts = layer.inspect("counts").cpu().numpy()

    # ---- device-timed region (inputs resident in HBM) ----
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index) as clk:
        e0.record(stream)
        for _ in range(steps):
            layer.forward(x, y, idx, gate)
        e1.record(stream)
        torch.cuda.synchronize(device)
    barrier()
    ms_max = max_over_ranks(e0.elapsed_time(e1), world, device)

    # ---- the same loop with the library's per-stage CUDA events (recorded on the launching stream
    #      between kernels): stage breakdown and the dominant kernel's launch duration.  The events
    #      lengthen a step by a few percent, which is why the headline loop runs without them ----
    layer.profile(True)
    barrier()
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(steps):
        layer.forward(x, y, idx, gate)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    layer.profile(False)
    prof_ms_max = max_over_ranks(e0.elapsed_time(e1), world, device)
    stage_ms, recorded, launches = layer.profile_read()
    if layer.device_status() != 0:
        raise RuntimeError("device status not clean after the timed region")

    # ---- end to end through the host-buffer entry point ----
    xh = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty((t, wl.shape.d), dtype=torch.bfloat16).pin_memory()
    ih = torch.empty((t, wl.shape.top_k), dtype=torch.int32).pin_memory()
    gh = torch.empty((t, wl.shape.top_k), dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(steps, 200))
    for _ in range(2):
        layer.forward_host(xh, yh, ih, gh)
    torch.cuda.synchronize(device)
    barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        layer.forward_host(xh, yh, ih, gh)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)

    work = algorithmic_work(wl, counts)
    pk, pk_kind = peaks()
    p_tc = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    tc_src = pk_kind + " bf16 (sustained)"
    if wl.precision == "nvfp4":  # no measured FP4 peak: bf16 measured x the nominal 4x FP4/BF16 ratio
        p_tc *= 4.0
        tc_src = pk_kind + " bf16 (sustained) x nominal FP4/BF16 ratio 4"
    # dominant kernel: the stage with the largest device time
    dom = max(stage_ms, key=stage_ms.get)
    per_launch_ms = stage_ms[dom] / max(1, recorded)
    decode_like = wl.tokens * wl.shape.top_k <= 48 * wl.shape.n_experts
    roof = None
    if dom in ("expert_up", "expert_down"):
        unit_work = work[dom]
        regime = "decode" if decode_like else ("prefill" if wl.tokens * wl.shape.top_k >= 256 * wl.shape.n_experts
                                                 else "skewed")
        ratio = TRAFFIC_RATIO.get((wl.precision, regime, dom))
        traffic = None
        if ratio is not None and gemm_sources_sha256() == TRAFFIC_SOURCES_SHA256:
            traffic = ratio * unit_work["bytes"]
        gbs = unit_work["bytes"] / (per_launch_ms * 1e-3) / 1e9
        tfs = unit_work["flops"] / (per_launch_ms * 1e-3) / 1e12
        both = {"hbm_frac": gbs / pk["hbm_gbs"], "tc_frac": tfs / p_tc}
        if decode_like:
            roof = {"kernel": dom, "bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / pk["hbm_gbs"], "traffic": traffic, "algorithmic_bytes": unit_work["bytes"],
                    "launch_ms": per_launch_ms, "peak_source": pk_kind, **both}
        else:
            roof = {"kernel": dom, "bound": "tensor", "achieved": tfs, "peak": p_tc, "unit": "TFLOP/s",
                    "frac": tfs / p_tc, "traffic": traffic, "algorithmic_flops": unit_work["flops"],
                    "algorithmic_bytes": unit_work["bytes"], "launch_ms": per_launch_ms, "peak_source": tc_src,
                    **both}
    step_ms = ms_max / steps
    lay = work["layer"]
    layer_roof = {"bytes_per_step": lay["bytes"], "flops_per_step": lay["flops"],
                  "hbm_frac": lay["bytes"] / (step_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                  "tc_frac_of_bf16_peak": lay["flops"] / (step_ms * 1e-3) / 1e12 /
                  pk.get("bf16_tflops_sustained", pk["bf16_tflops"])}
    out = {
        "value": whole_job_tokens_per_s(world, t, steps, ms_max),
        "unit": "tokens/s",
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": step_ms,
        "dtype": "nvfp4+bf16" if wl.precision == "nvfp4" else "bf16",
        "config": {"workload": wl.name, "tokens": t, "d": wl.shape.d, "latent": wl.shape.latent,
                   "experts": wl.shape.n_experts, "top_k": wl.shape.top_k, "expert_ffn": wl.shape.expert_ffn,
                   "shared_ffn": wl.shape.shared_ffn, "precision": wl.precision,
                   "parallelism": f"{world} independent replica(s)",
                   "l2": "inputs larger than L2: every step streams all touched expert weights "
                         f"({work['touched_experts']} experts, {work['expert_weight_bytes'] / 1e9:.2f} GB)"},
        "roofline": roof,
        "layer_roofline": layer_roof,
        "load": load_stats(counts, t),
        "stages_ms_per_step": {k: v / max(1, recorded) for k, v in stage_ms.items()},
        "profiled_ms_per_step": prof_ms_max / steps,
        "e2e": {"value": whole_job_tokens_per_s(world, t, e2e_steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": t * wl.shape.d * 2,
                "d2h_bytes_per_step": t * wl.shape.d * 2 + t * wl.shape.top_k * 8, "steps": e2e_steps},
        "gpu_launches": launches * steps,
        "clocks": clk.summary(),
    }
    if with_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, w)
    return out


# The default run covers both halves of the metric: the decode batch (T = 256) is the headline
# line, the prefill batch (T = 16384, the same layer's weights) its "prefill" object.
PREFILL_OF = {"decode": "prefill", "decode_nvfp4": "prefill_nvfp4"}


def run_ours(args, wl, rank, world):
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    pwl = inp.workload(PREFILL_OF[wl.name]) if (wl.name in PREFILL_OF and not args.no_prefill) else None
    layer, w = make_device_layer(wl, device, max_tokens=max(wl.tokens, pwl.tokens if pwl else 0))
    cpu = world == 1 and rank == 0 and not args.no_cpu_baseline
    line = {"metric": METRIC, "n_gpus": world, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "data": "synthetic: seeded N(0,1/fan_in) weights, N(0,1) x, bf16" +
                    (" (experts and shared expert quantised to NVFP4 on the device)" if wl.precision == "nvfp4"
                     else "")}
    line.update(measure(layer, w, wl, args.steps, args.warmup, world, device, cpu))
    if pwl is not None:
        psteps = min(args.steps, DEFAULT_STEPS[pwl.name])
        p = measure(layer, w, pwl, psteps, args.warmup, world, device, cpu)
        line["prefill"] = p
        line["gpu_launches"] += p["gpu_launches"]
    layer.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode", choices=sorted(inp.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="decode workloads only: skip the prefill half of the line")
    args = ap.parse_args()
    wl = inp.workload(args.workload)
    if args.steps is None:
        args.steps = DEFAULT_STEPS.get(args.workload, DEFAULT_STEPS.get(args.workload.split("_")[0], 20))
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, wl, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
