"""Exact pins of the oracle's NVFP4 arithmetic (CPU only).

Source: "Drama 3 - NVFP4 routed experts", section "Quantization": E2M1 codes,
one E4M3 scale per 16 input channels, an FP32 global scale per matrix (gate
and up share it) and dynamic per-token activation scales.  The block-scaled
product of two NVFP4 operands is, by definition, the sum over channels of
E2M1(a) * S_a * E2M1(w) * S_w, times the two globals.

The E2M1 and E4M3 decode tables these tests use are themselves pinned
exhaustively in test_oracle_formats.py, so every expected value here comes
from the format definitions, not from the function under test.

- orc_nvfp4_global: hand values (amax 2688 gives 1, all-zero gives 1, ...).
- orc_nvfp4_gemv: constant-code closed form, a one-hot code per row with a
  distinct scale per (row, block) (fails any scale- or code-indexing slip),
  and a float64 matmul of the decoded operands within the fp32 summation
  bound.
- orc_expert_ffn_nvfp4: a closed form from constant codes with different
  gate and up values, and a stage-wise composition from the pinned pieces
  (x quantised, the gate/up GEMV, SwiGLU, h re-quantised, the down GEMV).
"""
import numpy as np
import pytest

import oracle
import synth

E2M1_ONE, E2M1_TWO, E2M1_HALF, E2M1_SIX, E2M1_ONE_HALF = 2, 4, 1, 7, 3
E4M3_ONE, E4M3_TWO, E4M3_HALF, E4M3_448 = 0x38, 0x40, 0x30, 0x7E
BF16_ONE = 0x3F80


def decode_operand(codes, sf):
    """E2M1 codes [N][K] with E4M3 scales [N][K/16] -> float64 values."""
    return (oracle.e2m1_to_f32(codes).astype(np.float64)
            * np.repeat(oracle.e4m3_to_f32(sf).astype(np.float64), 16, axis=-1))


# ------------------------------------------------------------------ global scale
def test_global_hand_values():
    v = np.zeros(100, np.float32)
    assert oracle.nvfp4_global(v) == 1.0            # all zero: 1 by definition
    v[17] = 2688.0
    assert oracle.nvfp4_global(v) == 1.0            # amax / (448 * 6)
    v[3] = -5376.0
    assert oracle.nvfp4_global(v) == 2.0            # amax of magnitudes
    v = np.full(7, 0.5, np.float32)
    v[2] = -1.0
    assert oracle.nvfp4_global(v) == np.float32(1.0) / np.float32(2688.0)


# ------------------------------------------------------------------ block-scaled GEMV
def test_gemv_constant_codes_closed_form():
    N, K = 32, 256
    a_c = np.full(K, E2M1_ONE, np.uint8)
    a_s = np.full(K // 16, E4M3_TWO, np.uint8)
    w_c = np.full((N, K), E2M1_TWO, np.uint8)
    w_s = np.full((N, K // 16), E4M3_HALF, np.uint8)
    y = oracle.nvfp4_gemv(a_c, a_s, 0.5, w_c, w_s, 0.25)
    # K * (1 * 2) * (2 * 0.5) * 0.5 * 0.25, exact in fp32
    assert np.all(y == np.float32(K * 2.0 * 1.0 * 0.125))
    a_c[:] = 8 | E2M1_ONE                            # sign bit: -1
    y = oracle.nvfp4_gemv(a_c, a_s, 0.5, w_c, w_s, 0.25)
    assert np.all(y == np.float32(-K * 0.25))


def test_gemv_one_hot_rows_with_distinct_row_block_scales():
    """Row n has one nonzero code, at column pi(n); every (row, block) has its
    own scale.  y[n] is one product, exact in fp32, so the check is equality;
    reading another row's scales, another block's scale, the transposed code
    or dropping a global changes it."""
    rng = np.random.default_rng(11)
    N, K = 48, 256
    a_c = rng.integers(0, 16, K).astype(np.uint8)
    a_c[a_c % 8 == 0] = 5                            # no zero activations
    a_s = rng.integers(0x28, 0x50, K // 16).astype(np.uint8)
    pi = rng.integers(0, K, N)
    w_c = np.zeros((N, K), np.uint8)
    w_c[np.arange(N), pi] = rng.integers(1, 8, N) | (rng.integers(0, 2, N) << 3)
    w_s = rng.integers(0x20, 0x60, (N, K // 16)).astype(np.uint8)
    Ga, Gw = 0.125, 4.0
    y = oracle.nvfp4_gemv(a_c, a_s, Ga, w_c, w_s, Gw)
    A = decode_operand(a_c, a_s)
    W = decode_operand(w_c, w_s)
    want = A[pi] * W[np.arange(N), pi] * Ga * Gw
    assert np.array_equal(y.astype(np.float64), want)


def test_gemv_float64_cross_check_within_fp32_sum_bound():
    rng = np.random.default_rng(5)
    N, K = 64, 2048
    a_c = rng.integers(0, 16, K).astype(np.uint8)
    a_s = rng.integers(0x20, 0x58, K // 16).astype(np.uint8)
    w_c = rng.integers(0, 16, (N, K)).astype(np.uint8)
    w_s = rng.integers(0x20, 0x58, (N, K // 16)).astype(np.uint8)
    Ga, Gw = np.float32(0.0123), np.float32(3.7e-4)
    y = oracle.nvfp4_gemv(a_c, a_s, Ga, w_c, w_s, Gw).astype(np.float64)
    A = decode_operand(a_c, a_s)
    W = decode_operand(w_c, w_s)
    g = float(np.float32(Ga) * np.float32(Gw))       # the oracle multiplies the globals in fp32
    ref = (W @ A) * g
    mag = (np.abs(W) @ np.abs(A)) * g
    # every product is exact in fp32 (at most 12 significant bits); the K-term
    # fp32 sum and the two final roundings stay within (K + 2) units of 2^-24
    bound = (K + 2) * 2.0 ** -24 * mag
    assert np.all(np.abs(y - ref) <= bound)
    assert np.max(np.abs(y - ref) / mag) < 1e-5


# ------------------------------------------------------------------ quantiser indexing
def test_quantize_per_row_block_scales_and_codes():
    """Blocks built so that scale and codes are known: block (n, b) holds
    6 * S[n][b] * G at one position and S[n][b] * G times a known code
    elsewhere."""
    rng = np.random.default_rng(3)
    N, K, G = 8, 64, np.float32(0.5)
    S = rng.integers(0x30, 0x60, (N, K // 16)).astype(np.uint8)
    Sf = oracle.e4m3_to_f32(S).astype(np.float32)
    codes = rng.integers(0, 16, (N, K)).astype(np.uint8)
    codes[:, ::16] = E2M1_SIX                        # each block's max magnitude is 6 S G
    v = (oracle.e2m1_to_f32(codes) * np.repeat(Sf, 16, 1) * G).astype(np.float32)
    c2, s2 = oracle.nvfp4_quantize(v, G)
    assert np.array_equal(s2, S)
    dec_want = oracle.e2m1_to_f32(codes)
    assert np.array_equal(oracle.e2m1_to_f32(c2), dec_want)  # +0 and -0 decode equal


# ------------------------------------------------------------------ expert FFN
def _const_layer(H, F, gate_code, up_code, down_code, G_gu, G_d):
    gu_c = np.empty((2 * F, H), np.uint8)
    gu_c[:F] = gate_code
    gu_c[F:] = up_code
    gu_s = np.full((2 * F, H // 16), E4M3_ONE, np.uint8)
    d_c = np.full((H, F), down_code, np.uint8)
    d_s = np.full((H, F // 16), E4M3_ONE, np.uint8)
    return (gu_c, gu_s, G_gu), (d_c, d_s, G_d)


def test_ffn_constant_codes_closed_form():
    """x = 1 everywhere quantises to code 6 with block scale 448 and global
    1/2688 (value 1).  Gate codes 0.5 and up codes 1.5 with G_gu = 2^-6 give
    g = H * 0.5 / 64 and u = H * 1.5 / 64; h = SiLU(g) * u is the same for
    every feature, so it re-quantises to code 6 and scale 448 again, and the
    down projection with codes 1 and G_d = 2^-9 gives Y = F * h / 512."""
    H, F = 256, 128
    gu, d = _const_layer(H, F, E2M1_HALF, E2M1_ONE_HALF, E2M1_ONE, 2.0 ** -6, 2.0 ** -9)
    x = np.full(H, BF16_ONE, np.uint16)
    Y, (h, hc, hs, hG) = oracle.expert_ffn_nvfp4(x, gu, d, stages=True)
    g, u = H * 0.5 / 64, H * 1.5 / 64
    h_want = g / (1 + np.exp(-g)) * u
    np.testing.assert_allclose(h, h_want, rtol=2e-6)
    assert np.all(hc == E2M1_SIX) and np.all(hs == E4M3_448)
    assert hG == np.float32(h[0]) / np.float32(2688.0)
    np.testing.assert_allclose(Y, F * h_want / 512, rtol=4e-6)
    # SiLU applies to the gate (rows [0, F)), not to the up rows
    gu_sw, _ = _const_layer(H, F, E2M1_ONE_HALF, E2M1_HALF, E2M1_ONE, 2.0 ** -6, 2.0 ** -9)
    Y2 = oracle.expert_ffn_nvfp4(x, gu_sw, d)
    np.testing.assert_allclose(Y2, F * (u / (1 + np.exp(-u)) * g) / 512, rtol=4e-6)


def test_ffn_stagewise_composition_of_pinned_pieces():
    H, F = 512, 256
    wg = synth.expert_weights(21, 0, 0, synth.PROJ_GATE_UP, 2 * F, H)
    wd = synth.expert_weights(21, 0, 0, synth.PROJ_DOWN, H, F)
    Ggu, Gd = oracle.nvfp4_global(wg), oracle.nvfp4_global(wd)
    gu = (*oracle.nvfp4_quantize(wg, Ggu), Ggu)
    d = (*oracle.nvfp4_quantize(wd, Gd), Gd)
    for t in range(3):
        x = synth.activations_bf16(21, t, 1, H)[0]
        Y, (h, hc, hs, hG) = oracle.expert_ffn_nvfp4(x, gu, d, stages=True)
        xf = synth.bf16_bits_to_f32(x).astype(np.float32)[None, :]
        Gx = oracle.nvfp4_global(xf)
        xc, xs = oracle.nvfp4_quantize(xf, Gx)
        gu_out = oracle.nvfp4_gemv(xc[0], xs[0], Gx, *gu)
        g, u = gu_out[:F].astype(np.float32), gu_out[F:].astype(np.float32)
        h_np = g / (np.float32(1) + np.exp(-g)) * u
        np.testing.assert_allclose(h, h_np, rtol=1e-6, atol=1e-30)
        Gh = oracle.nvfp4_global(h)
        assert hG == Gh
        hc2, hs2 = oracle.nvfp4_quantize(h[None, :], Gh)
        assert np.array_equal(hc, hc2[0]) and np.array_equal(hs, hs2[0])
        assert np.array_equal(Y, oracle.nvfp4_gemv(hc, hs, hG, *d))
        assert np.array_equal(Y, oracle.down_nvfp4(hc, hs, hG, d))
