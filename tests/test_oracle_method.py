"""Pins of the oracle's method functions (CPU only).

Quantiser: error bound and range coverage.  Dequant: hand-set values and the
single-rounding property.  Route: brute-force stable sort, k = 1, k = E, the
softmax-of-selected identity, ties.  Permute: brute-force stable sort.  FFN:
closed forms from hand-set codes and a float64 library cross-check.
Combine: one-hot weights and the dense-vs-sparse identity.  NVFP4: round
trips and error magnitude.
"""
import math

import numpy as np
import pytest

import oracle
import synth

F16_ONE, F16_HALF, F16_M8, F16_MAX, F16_TINY = 0x3C00, 0x3800, 0xC800, 0x7BFF, 0x0001


# ------------------------------------------------------------------ quantizer
def test_quantizer_error_bound_and_coverage():
    w = synth.expert_weights(11, 0, 3, synth.PROJ_GATE_UP, 64, 2048)
    codes, s_bits, m_bits = oracle.quantize_w4(w)
    s = s_bits.view(np.float16).astype(np.float64)
    m = m_bits.view(np.float16).astype(np.float64)
    g = w.reshape(64, 32, 64).astype(np.float64)
    # directed f16 roundings: [m, m + 15 s] covers [min, max] of each group
    assert np.all(m <= g.min(-1))
    assert np.all(m + 15 * s >= g.max(-1))
    wh = oracle.dequant_w4(codes, s_bits, m_bits).reshape(64, 32, 64).astype(np.float64)
    err = np.abs(wh - g)
    bound = s[..., None] / 2 + np.abs(g) * 2.0 ** -22 + 1e-12
    assert np.all(err <= bound)
    assert codes.max() == 15 and codes.min() == 0
    rel = np.linalg.norm(wh - g) / np.linalg.norm(g)
    assert 0.06 < rel < 0.11, rel  # uniform-step error of a 16-level grid over the group range


def test_quantizer_constant_and_closed_form_groups():
    w = np.zeros((2, 128), np.float32)
    w[0, :64] = 0.25            # constant group: scale 0, codes 0, min = f16 below 0.25
    w[0, 64:] = np.linspace(-1, 2, 64, dtype=np.float32)
    w[1, :64] = np.arange(64) % 16  # integers 0..15: min 0, scale exactly 1
    w[1, 64:] = -3.0
    codes, s, m = oracle.quantize_w4(w)
    assert s[0, 0] == 0 and m[0, 0] == np.float16(0.25).view(np.uint16) and codes[0, :64].max() == 0
    assert s[1, 0] == F16_ONE and m[1, 0] == 0
    assert np.array_equal(codes[1, :64], (np.arange(64) % 16).astype(np.uint8))
    assert s[1, 1] == 0 and m[1, 1] == np.float16(-3.0).view(np.uint16)
    # range [-1, 2]: min exactly -1, scale = f16 above 3/15
    assert m[0, 1] == np.float16(-1.0).view(np.uint16)
    sc = float(np.float16(0.2))
    want = sc if sc >= 0.2 else float(np.nextafter(np.float16(0.2), np.float16(1)))
    assert float(s[0, 1].view(np.float16)) == want
    assert codes[0, 64] == 0 and codes[0, 127] == 15


# ------------------------------------------------------------------ packing / dequant
def test_canonical_pack_round_trip_and_nibble_order():
    rng = np.random.default_rng(2)
    for codes in [rng.integers(0, 16, (16, 128)), np.zeros((16, 128)), np.full((16, 128), 15),
                  np.tile([0, 15], (16, 64))]:
        codes = codes.astype(np.uint8)
        words = oracle.pack_nibbles(codes)
        assert np.array_equal(oracle.unpack_nibbles(words, 128), codes)
    one = np.arange(8, dtype=np.uint8)[None, :]
    assert int(oracle.pack_nibbles(one)[0, 0]) == 0x76543210


def test_dequant_hand_set_values():
    assert oracle.dequant_one(15, F16_ONE, F16_M8) == 7.0
    assert oracle.dequant_one(1, F16_HALF, 0) == 0.5
    assert oracle.dequant_one(9, 0, F16_M8) == -8.0
    assert oracle.dequant_one(1, F16_MAX, 0) == 65504.0
    assert oracle.dequant_one(15, F16_TINY, 0) == 15 * 2.0 ** -24


def test_dequant_is_one_rounding_of_the_exact_value():
    rng = np.random.default_rng(3)
    s = rng.integers(0x0400, 0x3000, 3000).astype(np.uint16)
    m = (rng.integers(0x0400, 0x3000, 3000) | (rng.integers(0, 2, 3000) << 15)).astype(np.uint16)
    q = rng.integers(0, 16, 3000)
    exact = q * s.view(np.float16).astype(np.float64) + m.view(np.float16).astype(np.float64)
    got = np.array([oracle.dequant_one(a, b, c) for a, b, c in zip(q, s, m)], np.float32)
    assert np.array_equal(got, exact.astype(np.float32))


# ------------------------------------------------------------------ routing
def _brute_route(l, k):
    order = sorted(range(len(l)), key=lambda e: (-float(l[e]), e))
    sel = order[:k]
    ls = np.array([float(l[e]) for e in sel])
    p = np.exp(ls - ls.max())
    return sel, p / p.sum()


@pytest.mark.parametrize("T,E,k,tie", [(4, 8, 2, False), (16, 256, 8, False), (16, 256, 8, True),
                                       (3, 64, 6, True)])
def test_route_brute_force(T, E, k, tie):
    l = synth.router_logits(5, 0, T, E, bf16_rounded=tie)
    if tie:
        l = np.round(l * 4) / 4  # many exact ties
    idx, w = oracle.route(l, k)
    for t in range(T):
        sel, wr = _brute_route(l[t], k)
        assert list(idx[t]) == sel
        np.testing.assert_allclose(w[t], wr, rtol=2e-6)


def test_route_k1_kE_and_ties():
    l = synth.router_logits(6, 0, 5, 32)
    idx, w = oracle.route(l, 1)
    assert np.array_equal(idx[:, 0], np.argmax(l, axis=1)) and np.all(w == 1.0)
    idx, w = oracle.route(l, 32)
    full = np.exp(l - l.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    for t in range(5):
        np.testing.assert_allclose(w[t], full[t][idx[t]], rtol=2e-6)
        assert abs(float(w[t].sum()) - 1) < 32 * 2 ** -23
    eq = np.zeros((2, 8), np.float32)
    idx, w = oracle.route(eq, 3)
    assert idx.tolist() == [[0, 1, 2], [0, 1, 2]] and np.allclose(w, 1 / 3)
    idx, _ = oracle.route(np.array([[1, 3, 3, 2]], np.float32), 2)
    assert idx.tolist() == [[1, 2]]


# ------------------------------------------------------------------ permutation
@pytest.mark.parametrize("T,k,E", [(4, 2, 8), (2048, 8, 256), (0, 8, 256), (17, 3, 4)])
def test_permute_brute_force(T, k, E):
    rng = np.random.default_rng(T)
    if T:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    else:
        idx = np.zeros((0, k), np.int32)
    counts, offsets, sorted_rows, inv = oracle.permute(idx, E)
    flat = idx.ravel()
    order = sorted(range(T * k), key=lambda r: (int(flat[r]), r))
    assert sorted_rows.tolist() == order
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k and np.all(np.diff(offsets) == counts)
    assert np.array_equal(sorted_rows[inv], np.arange(T * k))


# ------------------------------------------------------------------ expert FFN
def _silu(g):
    return g / (1.0 + math.exp(-g))


def test_ffn_constant_codes_closed_form():
    H, F = 128, 64
    x = synth.activations_bf16(1, 0, 1, H)[0]
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    cg, s, m = 5, np.float16(0.01).view(np.uint16), np.float16(-0.03).view(np.uint16)
    gu = (np.full((2 * F, H), cg, np.uint8), np.full((2 * F, H // 64), s, np.uint16),
          np.full((2 * F, H // 64), m, np.uint16))
    d = (np.full((H, F), 9, np.uint8), np.full((H, 1), s, np.uint16), np.full((H, 1), m, np.uint16))
    Y, h = oracle.expert_ffn_w4(x, gu, d, return_h=True)
    w0 = 5 * float(np.float16(0.01)) + float(np.float16(-0.03))
    wd = 9 * float(np.float16(0.01)) + float(np.float16(-0.03))
    g = w0 * xf.sum()
    np.testing.assert_allclose(h, _silu(g) * g, rtol=1e-5)
    np.testing.assert_allclose(Y, wd * F * _silu(g) * g, rtol=1e-5)


def test_ffn_permutation_codes_closed_form():
    H, F = 128, 64
    rng = np.random.default_rng(4)
    x = synth.activations_bf16(2, 0, 1, H)[0]
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    pg, pu, pd = rng.permutation(H)[:F], rng.permutation(H)[:F], rng.integers(0, F, H)
    codes = np.zeros((2 * F, H), np.uint8)
    codes[np.arange(F), pg] = 1
    codes[F + np.arange(F), pu] = 1
    dc = np.zeros((H, F), np.uint8)
    dc[np.arange(H), pd] = 1
    gu = (codes, np.full((2 * F, 2), F16_ONE, np.uint16), np.zeros((2 * F, 2), np.uint16))
    d = (dc, np.full((H, 1), F16_ONE, np.uint16), np.zeros((H, 1), np.uint16))
    Y, h = oracle.expert_ffn_w4(x, gu, d, return_h=True)
    hh = np.array([_silu(xf[pg[n]]) * xf[pu[n]] for n in range(F)])
    np.testing.assert_allclose(h, hh, rtol=1e-6, atol=1e-30)
    np.testing.assert_allclose(Y, hh[pd], rtol=1e-6, atol=1e-30)


def test_ffn_random_weights_float64_library_cross_check():
    H, F = 256, 128
    wg = synth.expert_weights(3, 0, 0, 0, 2 * F, H)
    wd = synth.expert_weights(3, 0, 0, 1, H, F)
    gu, d = oracle.quantize_w4(wg), oracle.quantize_w4(wd)
    x = synth.activations_bf16(3, 0, 1, H)[0]
    Y, h = oracle.expert_ffn_w4(x, gu, d, return_h=True)
    Wgu = oracle.dequant_w4(*gu).astype(np.float64)
    Wd = oracle.dequant_w4(*d).astype(np.float64)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    gu64 = Wgu @ xf
    h64 = gu64[:F] / (1 + np.exp(-gu64[:F])) * gu64[F:]
    Y64 = Wd @ h64
    assert np.linalg.norm(h - h64) / np.linalg.norm(h64) < 1e-5
    assert np.linalg.norm(Y - Y64) / np.linalg.norm(Y64) < 1e-5


# ------------------------------------------------------------------ combine / whole layer
def _tiny_layer(seed=0, E=8, H=128, F=64):
    return {e: (oracle.quantize_w4(synth.expert_weights(seed, 0, e, 0, 2 * F, H)),
                oracle.quantize_w4(synth.expert_weights(seed, 0, e, 1, H, F))) for e in range(E)}


def test_combine_one_hot_and_rounding():
    rows = synth.normal_f32(1, 9, 9, 3 * 2 * 64, 1.0).reshape(6, 64)
    w = np.array([[1, 0], [0, 1], [0.5, 0.5]], np.float32)
    y = oracle.combine(rows, w)
    assert np.array_equal(y[0], synth.f32_to_bf16_bits(rows[0]))
    assert np.array_equal(y[1], synth.f32_to_bf16_bits(rows[3]))
    assert np.array_equal(y[2], synth.f32_to_bf16_bits(0.5 * rows[4] + 0.5 * rows[5]))


def test_dense_over_all_experts_equals_sparse_topk():
    """sum_e wfull[e] * FFN_e(x) with wfull zero off the top-k equals the routed result."""
    E, k, H, F, T = 8, 2, 128, 64, 4
    experts = _tiny_layer()
    x = synth.activations_bf16(0, 0, T, H)
    logits = synth.router_logits(0, 0, T, E)
    idx, w, y_rows, y = oracle.moe_forward_w4(x, logits, k, experts)
    for t in range(T):
        wfull = np.zeros(E, np.float32)
        wfull[idx[t]] = w[t]
        allY = np.stack([oracle.expert_ffn_w4(x[t], *experts[e]) for e in range(E)])
        dense = np.zeros(H, np.float32)
        for e in range(E):
            dense += wfull[e] * allY[e]
        ysp = synth.bf16_bits_to_f32(y[t])
        np.testing.assert_allclose(ysp, dense, rtol=2 ** -7, atol=1e-6)
        for j in range(k):
            assert np.array_equal(y_rows[t * k + j], allY[idx[t, j]])


# ------------------------------------------------------------------ NVFP4
def test_nvfp4_round_trip_of_representable_values():
    rng = np.random.default_rng(7)
    G = 0.001
    sf = rng.integers(0x20, 0x70, (4, 8)).astype(np.uint8)  # E4M3 scales
    codes = rng.integers(0, 16, (4, 128)).astype(np.uint8)
    codes[:, ::16] = 7  # each block holds its max magnitude 6 so amax/6 = scale
    v = (oracle.e2m1_to_f32(codes) * np.repeat(oracle.e4m3_to_f32(sf), 16, 1)).astype(np.float32) * np.float32(G)
    c2, s2 = oracle.nvfp4_quantize(v, G)
    dec = oracle.e2m1_to_f32(c2) * np.repeat(oracle.e4m3_to_f32(s2), 16, 1) * np.float32(G)
    np.testing.assert_allclose(dec, v, rtol=1e-6, atol=0)


def test_nvfp4_weight_error_magnitude():
    w = synth.expert_weights(4, 0, 0, 0, 256, 512)
    G = oracle.nvfp4_global(w)
    c, s = oracle.nvfp4_quantize(w, G)
    dec = oracle.e2m1_to_f32(c) * np.repeat(oracle.e4m3_to_f32(s), 16, 1) * np.float32(G)
    rel = np.linalg.norm(dec - w) / np.linalg.norm(w)
    assert 0.06 < rel < 0.13, rel
    # every element within half a step of its block's grid (largest step 2 * S_b * G)
    step = 2 * np.repeat(oracle.e4m3_to_f32(s), 16, 1) * G
    assert np.all(np.abs(dec - w) <= step / 2 * (1 + 1e-5) + 1e-12)


def test_nvfp4_ffn_error_against_unquantized_is_order_0p2():
    """The NVFP4 canaries reported ~0.2 expert-output rel-L2; same order here."""
    H, F = 256, 128
    wg = synth.expert_weights(8, 0, 0, 0, 2 * F, H)
    wd = synth.expert_weights(8, 0, 0, 1, H, F)
    Ggu, Gd = oracle.nvfp4_global(wg), oracle.nvfp4_global(wd)
    gu = (*oracle.nvfp4_quantize(wg, Ggu), Ggu)
    d = (*oracle.nvfp4_quantize(wd, Gd), Gd)
    errs = []
    for t in range(4):
        x = synth.activations_bf16(8, t, 1, H)[0]
        Y = oracle.expert_ffn_nvfp4(x, gu, d)
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        g = wg.astype(np.float64) @ xf
        h = g[:F] / (1 + np.exp(-g[:F])) * g[F:]
        Yr = wd.astype(np.float64) @ h
        errs.append(np.linalg.norm(Y - Yr) / np.linalg.norm(Yr))
    assert 0.05 < np.mean(errs) < 0.4, errs
