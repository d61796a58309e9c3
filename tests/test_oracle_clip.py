"""Pins of the oracle's MSE clip-search quantisers and of the symmetric
group-128 int4 format (CPU only).

Sources: "Drama 3 int4 (drama-rs format)", table "What's quantized" (int4,
asymmetric, group 64, f16 scale + min, MSE clip search); "drama-3-w4a16",
section "How it was made" (round-to-nearest, one scale per 128 input
weights, each scale chosen from 20 clipping ratios 1.0 -> 0.81 by minimum
squared error; mean relative reconstruction error 10.3 %, about what int4
group-128 rounding gives on Gaussian weights) and table "At a glance" (int4,
symmetric, group 128, GPTQ packing).

- The clip search never does worse than the plain min/max quantiser (pinned
  in test_oracle_method.py), and its choice is the brute-force minimum of
  the 20 candidates' float64 squared errors.
- Codes are round-to-nearest for the chosen scale (error <= s/2 inside the
  range, clamped outside).
- Exactly representable groups come back unchanged; all-zero groups give
  scale 0.
- The mean relative error on Gaussian weights is the page's ~10.3 %.
- The symmetric group-128 FFN equals, bit for bit, the (pinned) asymmetric
  group-64 FFN of the same weights written as scale s and min -8 s.
"""
import os

import numpy as np
import pytest

import oracle
import synth

def _page_figure(key):
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_figures.txt")) as f:
        for line in f:
            parts = line.split("|")[0].split()
            if len(parts) == 2 and parts[0] == key:
                return float(parts[1])
    raise KeyError(key)


# the page's schedule: 20 ratios from 1.00 down to 0.81 in steps of 0.01
RATIOS = [np.float32(100 - i) / np.float32(100) for i in range(int(_page_figure("clip_ratio_count")))]
assert float(RATIOS[0]) == _page_figure("clip_ratio_first") and abs(float(RATIOS[-1]) - _page_figure("clip_ratio_last")) < 1e-6


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def group_err64(w, codes, s_bits, m_bits):
    N, K = w.shape
    deq = codes.reshape(N, K // 64, 64) * f16(s_bits)[..., None] + f16(m_bits)[..., None]
    return ((deq - w.reshape(N, K // 64, 64).astype(np.float64)) ** 2).sum(-1)


def group_err128(w, codes, s_bits):
    N, K = w.shape
    deq = (codes.reshape(N, K // 128, 128).astype(np.float64) - 8) * f16(s_bits)[..., None]
    return ((deq - w.reshape(N, K // 128, 128).astype(np.float64)) ** 2).sum(-1)


def f16_round(x, mode):
    return np.array([oracle.f32_to_f16(np.float32(v), mode) for v in np.ravel(x)], np.uint16).reshape(np.shape(x))


# ------------------------------------------------------------------ asymmetric group 64
def test_asym_clip_never_worse_than_min_max_and_is_the_candidate_minimum():
    w = synth.expert_weights(41, 0, 2, synth.PROJ_GATE_UP, 32, 512)
    c, s, m = oracle.quantize_w4_clip(w)
    c0, s0, m0 = oracle.quantize_w4(w)
    e_clip, e_plain = group_err64(w, c, s, m), group_err64(w, c0, s0, m0)
    assert np.all(e_clip <= e_plain * (1 + 1e-6))
    assert np.mean(e_clip) < np.mean(e_plain)  # the search does pick clipped ranges
    # brute force: every ratio's candidate (scaled range, same roundings), coded by nearest rounding
    g = w.reshape(32, 8, 64)
    mn, mx = g.min(-1), g.max(-1)
    best = np.full(mn.shape, np.inf)
    for p in RATIOS:
        mb = f16_round(p * mn, 1)
        mf = f16(mb).astype(np.float32)
        sb = f16_round((p * mx - mf) / np.float32(15), 2)
        sf = f16(sb).astype(np.float32)
        q = np.clip(np.rint((g - mf[..., None]) / np.where(sf > 0, sf, 1)[..., None]), 0, 15)
        q = np.where(sf[..., None] > 0, q, 0)
        deq = q * sf[..., None].astype(np.float64) + mf[..., None]
        best = np.minimum(best, ((deq - g) ** 2).sum(-1))
    np.testing.assert_allclose(e_clip, best, rtol=1e-5, atol=0)


def test_asym_clip_codes_are_nearest_for_the_chosen_range():
    w = synth.expert_weights(42, 0, 1, synth.PROJ_DOWN, 16, 256)
    c, s, m = oracle.quantize_w4_clip(w)
    sf, mf = np.repeat(f16(s), 64, 1), np.repeat(f16(m), 64, 1)
    deq = c * sf + mf
    inside = (w >= mf) & (w <= mf + 15 * sf)
    assert np.all(np.abs(deq - w)[inside] <= sf[inside] / 2 * (1 + 1e-6))
    assert np.all(c[w < mf] == 0) and np.all(c[w > mf + 15 * sf] == 15)


def test_asym_clip_exact_groups_and_zero_groups():
    s0, m0 = np.float32(2.0 ** -8), np.float32(-0.03125)  # f16-exact scale and min
    q = np.tile(np.arange(16), 4).astype(np.float32)
    w = np.stack([q * s0 + m0, np.zeros(64, np.float32)])
    c, s, m = oracle.quantize_w4_clip(w)
    assert np.array_equal(c[0], q.astype(np.uint8))
    assert f16(s[0, 0]) == s0 and f16(m[0, 0]) == m0
    assert f16(s[1, 0]) == 0 and np.all(c[1] == 0)


# ------------------------------------------------------------------ symmetric group 128
def test_sym128_dequant_hand_values():
    one, half = 0x3C00, 0x3800
    assert oracle.lib().orc_dequant_sym128(15, one) == 7.0
    assert oracle.lib().orc_dequant_sym128(0, half) == -4.0
    assert oracle.lib().orc_dequant_sym128(8, 0x7BFF) == 0.0
    assert oracle.lib().orc_dequant_sym128(9, 0x7BFF) == 65504.0


def test_sym128_choice_is_the_candidate_minimum_and_codes_are_nearest():
    w = synth.expert_weights(43, 0, 0, synth.PROJ_GATE_UP, 24, 512)
    c, s = oracle.quantize_sym128(w)
    err = group_err128(w, c, s)
    g = w.reshape(24, 4, 128)
    amax = np.abs(g).max(-1)
    best = np.full(amax.shape, np.inf)
    for p in RATIOS:
        sb = f16_round((np.float32(2) * (p * amax)) / np.float32(15), 0)
        sf = f16(sb).astype(np.float32)
        q = np.clip(np.rint(g / sf[..., None]) + 8, 0, 15)
        deq = (q - 8) * sf[..., None].astype(np.float64)
        best = np.minimum(best, ((deq - g) ** 2).sum(-1))
    np.testing.assert_allclose(err, best, rtol=1e-5, atol=0)
    sf = np.repeat(f16(s), 128, 1)
    deq = (c.astype(np.float64) - 8) * sf
    inside = (w >= -8 * sf) & (w <= 7 * sf)
    assert np.all(np.abs(deq - w)[inside] <= sf[inside] / 2 * (1 + 1e-6))
    assert np.all(c[w < -8 * sf] == 0) and np.all(c[w > 7 * sf] == 15)


def test_sym128_zero_group():
    c, s = oracle.quantize_sym128(np.zeros((1, 128), np.float32))
    assert s[0, 0] == 0 and np.all(c == 8)


def test_sym128_gaussian_error_matches_the_page():
    """The w4a16 page: mean relative reconstruction error per expert matrix
    10.3 %, about what int4 group-128 rounding gives on Gaussian weights."""
    rng = np.random.default_rng(2026)
    errs = []
    for _ in range(4):
        w = (rng.standard_normal((128, 1024)) * 0.02).astype(np.float32)
        c, s = oracle.quantize_sym128(w)
        deq = (c.astype(np.float64) - 8) * np.repeat(f16(s), 128, 1)
        errs.append(np.linalg.norm(deq - w) / np.linalg.norm(w))
    page = _page_figure("sym128_mean_rel_error")
    assert 0.92 * page < np.mean(errs) < 1.05 * page, errs


def test_sym128_ffn_equals_the_asymmetric_ffn_of_the_same_weights():
    """(q - 8) s is q * s + m with m = -8 s, exactly, and a group of 128 is two
    groups of 64 with the same scale: the pinned int4 FFN must agree bit for
    bit."""
    H, F = 256, 256  # two groups of 128 along both inputs
    wg = synth.expert_weights(44, 0, 0, synth.PROJ_GATE_UP, 2 * F, H)
    wd = synth.expert_weights(44, 0, 0, synth.PROJ_DOWN, H, F)
    gu, d = oracle.quantize_sym128(wg), oracle.quantize_sym128(wd)

    def as_asym(codes, s):
        s64 = np.repeat(s, 2, axis=1)
        m64 = np.array([oracle.f32_to_f16(np.float32(-8.0) * np.float32(f16(b)), 0) for b in s64.ravel()],
                       np.uint16).reshape(s64.shape)
        assert np.all(f16(m64) == -8 * f16(s64))
        return codes, s64, m64

    for t in range(3):
        x = synth.activations_bf16(44, t, 1, H)[0]
        Y, h = oracle.expert_ffn_sym128(x, gu, d, return_h=True)
        Y4, h4 = oracle.expert_ffn_w4(x, as_asym(*gu), as_asym(*d), return_h=True)
        assert np.array_equal(Y, Y4) and np.array_equal(h, h4)
        # and a float64 matmul of the dequantised weights
        Wg = (gu[0].astype(np.float64) - 8) * np.repeat(f16(gu[1]), 128, 1)
        Wd = (d[0].astype(np.float64) - 8) * np.repeat(f16(d[1]), 128, 1)
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        g = Wg @ xf
        h64 = g[:F] / (1 + np.exp(-g[:F])) * g[F:]
        np.testing.assert_allclose(Y, Wd @ h64, rtol=1e-4, atol=1e-5 * np.abs(Wd @ h64).max())
