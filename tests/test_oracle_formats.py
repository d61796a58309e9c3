"""Pins of the oracle's number formats and the seeded generator (CPU only).

Every check compares the oracle with something other than itself: numpy's and
torch's own conversions, the formats' closed-form value tables, published
known-answer vectors, or a brute-force search.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ generator
def test_philox_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(h, 16) for h in r]
        out = synth.philox4x32_10(*v[:6])
        assert [int(o) for o in out] == v[6:]


def test_generator_moments_and_determinism():
    a = synth.normal_f32(7, 3, 5, 200000, 0.02)
    b = synth.normal_f32(7, 3, 5, 200000, 0.02)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert abs(a.std() - 0.02) < 2e-4 and abs(a.mean()) < 2e-4
    # Irwin-Hall(4) is bounded by 2*sqrt(3) standard deviations
    assert np.abs(a).max() <= 0.02 * 2 * np.sqrt(3) * (1 + 1e-6)
    # offsets address the same stream
    c = synth.normal_f32(7, 3, 5, 100, 0.02, start=1000)
    assert np.array_equal(c, a[1000:1100])


def test_generator_c_twin_matches_numpy_definition():
    ref = synth.normal_f32_numpy(9, 4 * 17 + 1, 3, 50000, 0.02, start=2 ** 32 - 100)
    got = synth.normal_f32(9, 4 * 17 + 1, 3, 50000, 0.02, start=2 ** 32 - 100)
    assert np.array_equal(ref.view(np.uint32), got.view(np.uint32))


# ------------------------------------------------------------------ binary16
def test_f16_decode_exhaustive_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = oracle.f16_to_f32(bits)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def _f32_samples(n=40000, seed=0):
    rng = np.random.default_rng(seed)
    e = rng.uniform(-30, 18, n)
    v = (rng.uniform(1, 2, n) * 2.0 ** e * rng.choice([-1, 1], n)).astype(np.float32)
    # exact f16 values, midpoints and neighbours of them
    h = rng.integers(0, 0x7BFF, 4000).astype(np.uint16).view(np.float16).astype(np.float32)
    mids = (h.astype(np.float64) + np.nextafter(h.astype(np.float16), np.float16(np.inf)).astype(np.float64)) / 2
    extra = np.concatenate([h, -h, mids.astype(np.float32), [0.0, -0.0, 65504, 65519, 65520, 1e6, -1e6,
                                                          2 ** -24, 2 ** -25, 3 * 2 ** -26, 6e-8]])
    return np.concatenate([v, extra.astype(np.float32)])


def test_f16_nearest_even_matches_numpy():
    x = _f32_samples()
    got = oracle.f32_to_f16(x, 0)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("mode", [1, 2])
def test_f16_directed_rounding_brackets(mode):
    x = _f32_samples(seed=mode)
    x = x[np.abs(x) <= 65504]
    got = oracle.f32_to_f16(x, mode).view(np.float16)
    g64 = got.astype(np.float64)
    x64 = x.astype(np.float64)
    if mode == 1:  # toward -inf: largest f16 <= x
        assert np.all(g64 <= x64)
        nxt = np.nextafter(got, np.float16(np.inf)).astype(np.float64)
        assert np.all(nxt > x64)
    else:  # toward +inf: smallest f16 >= x
        assert np.all(g64 >= x64)
        prv = np.nextafter(got, np.float16(-np.inf)).astype(np.float64)
        assert np.all(prv < x64)


# ------------------------------------------------------------------ bfloat16
def test_bf16_nearest_even_matches_torch():
    x = _f32_samples(seed=5)
    got = oracle.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    # the generator's own rounding of activations agrees too
    assert np.array_equal(synth.f32_to_bf16_bits(x), ref)


# ------------------------------------------------------------------ FP8 E4M3 / FP4 E2M1
def test_e4m3_decode_exhaustive_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_to_f32(codes)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.all(np.isnan(got[~fin])) and (~fin).sum() == 2
    assert np.nanmax(got) == 448.0


def test_e4m3_encode_matches_torch_in_range_and_saturates():
    rng = np.random.default_rng(1)
    x = (rng.uniform(1, 2, 20000) * 2.0 ** rng.uniform(-12, 8.8, 20000)).astype(np.float32)
    x = np.concatenate([x, -x, [0.0]])
    vals = oracle.e4m3_to_f32(np.arange(256, dtype=np.uint8))
    vals = vals[np.isfinite(vals)]
    mids = ((np.sort(np.unique(vals))[1:] + np.sort(np.unique(vals))[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, vals]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    got = oracle.f32_to_e4m3(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)
    big = np.array([449, 463.9, 464, 500, 1e9, -1e9], np.float32)
    assert np.all(oracle.e4m3_to_f32(oracle.f32_to_e4m3(big)) == np.sign(big) * 448)


E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # exponent bias 1, one mantissa bit


def test_e2m1_decode_table():
    got = oracle.e2m1_to_f32(np.arange(16, dtype=np.uint8))
    assert list(got[:8]) == E2M1_VALUES
    assert list(-got[8:]) == E2M1_VALUES


def test_e2m1_encode_brute_force_nearest_even():
    grid = np.array(E2M1_VALUES)
    xs = np.concatenate([np.linspace(-7, 7, 2801), (grid[1:] + grid[:-1]) / 2,
                         -(grid[1:] + grid[:-1]) / 2]).astype(np.float32)
    got = oracle.f32_to_e2m1(xs)
    for x, c in zip(xs, got):
        a = min(abs(float(x)), 6.0)
        d = np.abs(grid - a)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (c & 7) == want, (x, c)
        assert (c >> 3) == (1 if np.signbit(x) else 0)
