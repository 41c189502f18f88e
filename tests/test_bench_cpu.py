"""bench.py's host-side accounting, without a GPU: the algorithmic work of the expert launches
(including the shared expert the library folds into them at decode sizes) and the rule that the
measured DRAM traffic is only reported for the GEMM sources it was captured from."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import lmoe_inputs as inp  # noqa: E402


def _all_touched(wl):
    return np.ones(wl.shape.n_experts)


def test_decode_bytes_count_weights_activations_and_the_folded_shared_expert():
    wl = inp.workload("decode")
    s, t = wl.shape, wl.tokens
    tk = t * s.top_k
    w = bench.algorithmic_work(wl, _all_touched(wl))
    w_exp = s.n_experts * s.expert_ffn * s.latent * 2
    shared_up = s.shared_ffn * s.d * 2 + t * s.d * 2 + t * s.shared_ffn * 2
    assert w["expert_up"]["bytes"] == w_exp + tk * s.latent * 2 + tk * s.expert_ffn * 2 + shared_up
    assert w["expert_up"]["flops"] == 2 * tk * s.expert_ffn * s.latent + 2 * t * s.shared_ffn * s.d
    # the down launch writes the shared expert's output in fp32
    shared_down = s.d * s.shared_ffn * 2 + t * s.shared_ffn * 2 + t * s.d * 4
    assert w["expert_down"]["bytes"] == w_exp + tk * s.expert_ffn * 2 + tk * s.latent * 2 + tk * 4 + shared_down
    assert w["touched_experts"] == s.n_experts


def test_prefill_launches_do_not_fold_the_shared_expert():
    wl = inp.workload("prefill")
    s = wl.shape
    tk = wl.tokens * s.top_k
    w = bench.algorithmic_work(wl, _all_touched(wl))
    assert w["expert_up"]["flops"] == 2 * tk * s.expert_ffn * s.latent


def test_nvfp4_counts_codes_and_block_scales():
    wl = inp.workload("decode_nvfp4")
    s = wl.shape
    w = bench.algorithmic_work(wl, _all_touched(wl))
    per_elem = 0.5 + 1 / 16
    assert w["expert_weight_bytes"] == int(2 * s.n_experts * s.expert_ffn * s.latent * per_elem)


def test_standard_moe_experts_work_in_d():
    wl = inp.workload("standard_decode")
    s = wl.shape
    w = bench.algorithmic_work(wl, _all_touched(wl))
    assert w["expert_weight_bytes"] == 2 * s.n_experts * s.expert_ffn * s.d * 2
    assert w["layer"]["flops"] > 0


def test_traffic_hash_is_deterministic_and_covers_the_gemm_sources(tmp_path, monkeypatch):
    h = bench.gemm_sources_sha256()
    assert len(h) == 64 and h == bench.gemm_sources_sha256()
    # changed code changes the hash (the bench then reports no traffic); comments do not
    csrc = tmp_path / "latentmoe_expert_layer_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.TRAFFIC_SOURCES:
        (csrc / f).write_bytes(open(os.path.join(ROOT, "latentmoe_expert_layer_b200", "csrc", f), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.gemm_sources_sha256() == h
    with open(csrc / bench.TRAFFIC_SOURCES[0], "a") as fh:   # a comment: same code
        fh.write("\n// a note\n/* another */\n")
    assert bench.gemm_sources_sha256() == h
    with open(csrc / bench.TRAFFIC_SOURCES[0], "a") as fh:   # changed code
        fh.write("\nconstexpr int kProbe = 1;\n")
    assert bench.gemm_sources_sha256() != h
