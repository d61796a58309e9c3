"""Numeric readings the GPU kernels rely on, checked on the CPU (no GPU).

The grouped prefill forms each dequantised weight q*s + m with one fp32 FMA,
v*s + (m - 2^K*s), where v = 2^K + q is the nibble OR-ed into an exponent
pattern (K = 7, 11 or 15).  These tests pin that arithmetic against the
oracle's dequant (fmaf(q, s, m)), using exact float64 emulation of each fp32
rounding:
- on the test distribution, N(0, 0.02) weights quantised by the oracle, the
  FMA form equals fmaf(q, s, m) exactly for every code and every K;
- in general its error is at most 2^-24 * 2^K * |s| (<= 2^-9 |s|).
"""
import numpy as np
import pytest

import oracle
import synth


def _f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


def _f16_bits_to_f64(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _fma_form(q, s, m, K):
    """fp32 v*s + c with v = 2^K + q and c = fl32(m - 2^K s), each fp32 step
    rounded once (float64 holds every intermediate exactly)."""
    v = 2.0 ** K + q                      # exact in fp32 (the magic float)
    c = _f32(m - 2.0 ** K * s)            # fmaf(-2^K, s, m): one rounding
    return _f32(v * s + c)                # fmaf(v, s, c): one rounding


def _exact(q, s, m):
    return _f32(q * s + m)                # fmaf(q, s, m), the format's dequant


@pytest.mark.parametrize("K", [7, 11, 15])
def test_fma_form_equals_the_dequant_on_test_weights(K):
    w = synth.expert_weights(11, 0, 3, 0, 256, 512)  # N(0, 0.02) rows, 8 groups each
    codes, sb, mb = oracle.quantize_w4(w)
    s = _f16_bits_to_f64(sb)[:, :, None]
    m = _f16_bits_to_f64(mb)[:, :, None]
    q = np.arange(16, dtype=np.float64)[None, None, :]
    got = _fma_form(q, s, m, K)
    want = _exact(q, s, m)
    assert np.array_equal(got, want)
    # and the oracle's own dequant of the actual codes agrees with the reference formula
    deq = oracle.dequant_w4(codes, sb, mb).astype(np.float64).reshape(codes.shape[0], -1, 64)
    ref = _exact(codes.astype(np.float64).reshape(codes.shape[0], -1, 64), s, m)
    assert np.array_equal(deq, ref)


@pytest.mark.parametrize("K", [7, 11, 15])
def test_fma_form_error_bound_on_adversarial_groups(K):
    rng = np.random.default_rng(K)
    # scales and mins drawn far apart in magnitude (the constant m - 2^K s then rounds)
    s = _f32(np.abs(rng.normal(size=4000)) * 2.0 ** rng.integers(-20, 4, 4000))
    s = _f16_bits_to_f64(np.asarray(s, np.float16).view(np.uint16))
    m = _f16_bits_to_f64(np.asarray(rng.normal(size=4000) * 2.0 ** rng.integers(-24, 8, 4000),
                                     np.float16).view(np.uint16))
    ok = np.isfinite(s) & np.isfinite(m) & (s > 0)
    s, m = s[ok][:, None], m[ok][:, None]
    q = np.arange(16, dtype=np.float64)[None, :]
    err = np.abs(_fma_form(q, s, m, K) - _exact(q, s, m))
    # one rounding of the constant (<= 2^-24 * 2^K s relative to its size, with the
    # constant's magnitude below 2^(K+1) s + |m|) plus the final rounding's difference
    bound = 2.0 ** -24 * (2.0 ** (K + 1) * s + np.abs(m)) + 2.0 ** -23 * np.abs(q * s + m)
    assert np.all(err <= bound)
    assert np.all(err <= 2.0 ** -9 * s + 2.0 ** -23 * (np.abs(q * s + m) + np.abs(m)))
