"""The oracle and the library against the figures the pages print
(tests/golden/page_figures.txt, each with its page and section).  CPU only.

- NVFP4: the oracle's expert FFN on the page's shapes (hidden 2048, expert
  width 512) with NVFP4 weights and activations has the expert-output error
  of the page's two canaries (about 0.2 relative L2).
- Symmetric group 128 with the 20-ratio clip search: the per-matrix
  reconstruction error on Gaussian weights is the page's mean, and below its
  maximum.
- The packed formats cost the page's 4.5 bits per weight; the model shape
  (layers x experts x projections) is the page's matrix count, and the bench
  workloads use it.
"""
import os

import numpy as np

import oracle
import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def figures():
    out = {}
    with open(os.path.join(HERE, "golden", "page_figures.txt")) as f:
        for line in f:
            line = line.split("|")[0].strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                out[k] = float(v)
    return out


P = figures()


def test_nvfp4_expert_output_error_is_the_canaries():
    H, F = 2048, 512
    errs = []
    for e in range(2):
        wg = synth.expert_weights(8, 0, e, synth.PROJ_GATE_UP, 2 * F, H)
        wd = synth.expert_weights(8, 0, e, synth.PROJ_DOWN, H, F)
        Ggu, Gd = oracle.nvfp4_global(wg), oracle.nvfp4_global(wd)
        gu = (*oracle.nvfp4_quantize(wg, Ggu), Ggu)
        d = (*oracle.nvfp4_quantize(wd, Gd), Gd)
        for t in range(2):
            x = synth.activations_bf16(8, t, 1, H)[0]
            Y = oracle.expert_ffn_nvfp4(x, gu, d)
            xf = synth.bf16_bits_to_f32(x).astype(np.float64)
            g = wg.astype(np.float64) @ xf
            h = g[:F] / (1 + np.exp(-g[:F])) * g[F:]
            Yr = wd.astype(np.float64) @ h
            errs.append(np.linalg.norm(Y - Yr) / np.linalg.norm(Yr))
    canary = (P["nvfp4_canary_decode_rel_l2"] + P["nvfp4_canary_prefill_rel_l2"]) / 2
    assert 0.8 * canary < np.mean(errs) < 1.25 * canary, errs
    assert all(0.6 * canary < e < 1.5 * canary for e in errs), errs


def test_sym128_clip_search_error_is_the_pages():
    rng = np.random.default_rng(2026)
    errs = []
    for _ in range(4):
        w = (rng.standard_normal((128, 1024)) * 0.02).astype(np.float32)
        c, s = oracle.quantize_sym128(w)
        sc = np.asarray(s, np.uint16).view(np.float16).astype(np.float64)
        deq = (c.astype(np.float64) - 8) * np.repeat(sc, int(P["sym128_group"]), 1)
        errs.append(np.linalg.norm(deq - w) / np.linalg.norm(w))
    assert 0.92 * P["sym128_mean_rel_error"] < np.mean(errs) < 1.05 * P["sym128_mean_rel_error"], errs
    assert max(errs) < P["sym128_max_rel_error"]


def test_clip_ratio_schedule_is_the_pages():
    n, first, last = int(P["clip_ratio_count"]), P["clip_ratio_first"], P["clip_ratio_last"]
    ratios = [(100 - i) / 100 for i in range(n)]  # the schedule the quantisers use (p_i = (100 - i) / 100)
    assert ratios[0] == first and abs(ratios[-1] - last) < 1e-12


def test_packed_formats_cost_the_pages_bits_per_weight():
    import quantized_moe_route_b200 as moe
    for N, K in ((1024, 2048), (2048, 512)):
        assert moe.moe_nvfp4_packed_bytes(N, K) * 8 / (N * K) == P["nvfp4_bits_per_weight"]
        assert moe.moe_w4_packed_bytes(N, K) * 8 / (N * K) == P["nvfp4_bits_per_weight"]  # int4 g64: same 36 B / 64


def test_model_shape_is_the_pages():
    import sys
    sys.path.insert(0, os.path.dirname(HERE))
    import bench
    assert P["layers"] * P["routed_experts"] * P["projections"] == P["quantized_matrices"]
    assert bench.LAYERS == P["layers"] and bench.E == P["routed_experts"]
