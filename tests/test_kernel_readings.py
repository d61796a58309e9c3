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


# --------------------------------------------------------------- bit tricks
def _f32_from_bits(u):
    return np.asarray(u, np.uint32).view(np.float32).astype(np.float64)


def test_prefill_nibble_to_magic_float():
    """The prefill's per-word code extraction: for a packed word w, with
    wl = w << 8 and wr = w >> 12, pair i = 0..3 takes nibble i (channel k) and
    nibble i + 4 (channel k + 1) from (source, bit) = (wl, 8), (w, 16) for i = 0;
    (wl, 12), (wr, 8); (w, 8), (wr, 12); (w, 12), (wr, 16); OR-ed into the
    exponent pattern (150 - p) << 23 each is the fp32 value 2^(23 - p) + q."""
    rng = np.random.default_rng(0)
    w = rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32)
    wl = (w.astype(np.uint64) << 8).astype(np.uint32)
    wr = w >> 12
    src = {"w": w, "wl": wl, "wr": wr}
    plan = [(("wl", 8), ("w", 16)), (("wl", 12), ("wr", 8)), (("w", 8), ("wr", 12)), (("w", 12), ("wr", 16))]
    for i, pair in enumerate(plan):
        for odd, (name, p) in enumerate(pair):
            n = i + 4 * odd
            q = (w >> (4 * n)) & 15
            v = _f32_from_bits((src[name] & np.uint32(0xF << p)) | np.uint32((150 - p) << 23))
            assert np.array_equal(v, 2.0 ** (23 - p) + q), (i, odd)


def test_decode_int4_fragment_is_bf16_128_plus_q():
    """The int4 decode's A fragment: ((w >> 4 i) & 0x000F000F) | 0x43004300 holds,
    in each 16-bit half, the bf16 value 128 + q of nibble i (low half) and
    nibble i + 4 (high half)."""
    rng = np.random.default_rng(1)
    w = rng.integers(0, 2 ** 32, 5000, dtype=np.uint64).astype(np.uint32)
    for i in range(4):
        a = ((w >> (4 * i)) & np.uint32(0x000F000F)) | np.uint32(0x43004300)
        lo = _f32_from_bits((a & np.uint32(0xFFFF)) << 16)
        hi = _f32_from_bits(a & np.uint32(0xFFFF0000))
        assert np.array_equal(lo, 128.0 + ((w >> (4 * i)) & 15))
        assert np.array_equal(hi, 128.0 + ((w >> (4 * i + 16)) & 15))


@pytest.mark.parametrize("SH", [0, 4])
def test_decode_e2m1_pair_to_f16(SH):
    """The NVFP4 decode's fragment half: for the E2M1 codes at bits [SH, SH+4)
    and [SH+16, SH+20) of w, (sign * 2^(12 - SH)) + ((w << (9 - SH)) & 0x0E000E00)
    with sign = w & (0x00080008 << SH) is, per 16-bit half, the f16 encoding of
    the code's value times 2^-14 (E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6)."""
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    codes = np.arange(256, dtype=np.uint32)
    w = ((codes & 15) << SH) | ((codes >> 4) << (SH + 16))
    sgn = w & np.uint32(0x00080008 << SH)
    r = (sgn.astype(np.uint64) * (1 << (12 - SH)) + ((w.astype(np.uint64) << (9 - SH)) & 0x0E000E00)).astype(np.uint32)
    for half, c in ((r & np.uint32(0xFFFF), codes & 15), (r >> 16, codes >> 4)):
        val = half.astype(np.uint16).view(np.float16).astype(np.float64)
        want = np.where(c & 8, -1.0, 1.0) * e2m1[c & 7] * 2.0 ** -14
        assert np.array_equal(np.abs(val), np.abs(want))
        assert np.array_equal(np.signbit(val), (c & 8) != 0)


# --------------------------------------------------------------- tile schedule
def _cta_tile(i, b, G):
    """The prefill kernels' i-th tile of CTA b: passes of G tiles, alternately
    in and against CTA order."""
    return i * G + (G - 1 - b if i & 1 else b)


@pytest.mark.parametrize("G", [1, 2, 7, 148, 160])
def test_alternating_passes_cover_every_tile_once(G):
    """Each role of a CTA walks its tiles while cta_tile(i) < ntiles and stops at
    the first one past the end; over all CTAs that must visit every tile exactly
    once (no later pass may bring a CTA back below ntiles)."""
    for ntiles in list(range(0, 3 * G + 3)) + [560, 1120, 4321]:
        seen = []
        for b in range(G):
            i = 0
            while _cta_tile(i, b, G) < ntiles:
                seen.append(_cta_tile(i, b, G))
                i += 1
            # nothing below ntiles after the stop
            assert all(_cta_tile(j, b, G) >= ntiles for j in range(i, i + 4))
        assert sorted(seen) == list(range(ntiles))


def _chunks_int4_prefill(counts, BN=256, BM=128):
    """The int4 prefill's chunk numbering: per expert n // BN full chunks plus a
    partial one; chunks of more than BM rows ("heavy") first, then those of at
    most BM rows, each group in expert order.  Returns (e, row0, nvalid) per
    chunk index."""
    offsets = np.concatenate([[0], np.cumsum(counts)])
    hc = [n // BN + (1 if n % BN > BM else 0) for n in counts]
    lc = [1 if 0 < n % BN <= BM else 0 for n in counts]
    hs = np.concatenate([[0], np.cumsum(hc)])
    ls = np.concatenate([[0], np.cumsum(lc)])
    out = []
    for c in range(hs[-1] + ls[-1]):
        if c < hs[-1]:
            e = int(np.searchsorted(hs, c, side="right") - 1)
            row0 = offsets[e] + (c - hs[e]) * BN
        else:
            e = int(np.searchsorted(ls, c - hs[-1], side="right") - 1)
            row0 = offsets[e] + counts[e] // BN * BN
        out.append((e, int(row0), int(min(BN, offsets[e + 1] - row0))))
    return out, int(hs[-1])


def test_heavy_first_chunks_partition_the_rows():
    rng = np.random.default_rng(7)
    cases = [[0, 1, 127, 128, 129, 255, 256, 257, 384, 385, 513, 16], [0] * 5, [2048]]
    cases += [list(rng.integers(0, 700, rng.integers(1, 40))) for _ in range(50)]
    for counts in cases:
        chunks, nheavy = _chunks_int4_prefill(counts)
        offsets = np.concatenate([[0], np.cumsum(counts)])
        covered = np.zeros(int(offsets[-1]), np.int32)
        for c, (e, row0, nv) in enumerate(chunks):
            assert nv > 0 and offsets[e] <= row0 and row0 + nv <= offsets[e + 1]
            assert (nv > 128) == (c < nheavy)  # heavy chunks are exactly the first nheavy
            covered[row0:row0 + nv] += 1
        assert np.all(covered == 1)
