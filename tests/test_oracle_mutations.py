"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one small, plausible mistake in a copy of
oracle/moe_oracle.c: a dropped term, a wrong index, a swapped operand, a
wrong constant, a flipped comparison.  It compiles that copy with the
oracle's own flags and runs the pin tests against it in a child process
(ORACLE_LIB points the oracle wrapper at the broken build).  The test passes
only if some pin fails.  The real oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")
NVFP4_PINS = "tests/test_oracle_nvfp4.py"
METHOD_PINS = "tests/test_oracle_method.py"
CLIP_PINS = "tests/test_oracle_clip.py"
ROUTER_PINS = "tests/test_oracle_router.py"
SHARED_PINS = "tests/test_oracle_shared.py"

# (name, text in the oracle, replacement, pin file that must fail)
MUTATIONS = [
    ("nvfp4 gemv: row 0's block scales for every row",
     "w_sf[(size_t)n * (K / 16) + k / 16]", "w_sf[k / 16]", NVFP4_PINS),
    ("nvfp4 gemv: activation scale of the wrong block",
     "orc_e4m3_to_f32(a_sf[k / 16])", "orc_e4m3_to_f32(a_sf[k / 32])", NVFP4_PINS),
    ("nvfp4 gemv: weight operand transposed",
     "w_codes[(size_t)n * K + k]", "w_codes[(size_t)k * N + n]", NVFP4_PINS),
    ("nvfp4 gemv: weight global dropped",
     "y[n] = acc * (Ga * Gw);", "y[n] = acc * Ga;", NVFP4_PINS),
    ("nvfp4 global: 448 instead of 448 * 6",
     "return amax / 2688.0f;", "return amax / 448.0f;", NVFP4_PINS),
    ("nvfp4 global: zero tensor gives 0",
     "if (amax == 0.0f) return 1.0f;\n  return amax / 2688.0f;",
     "if (amax == 0.0f) return 0.0f;\n  return amax / 2688.0f;", NVFP4_PINS),
    ("nvfp4 quantiser: block scale without the factor 6",
     "const float denom = 6.0f * G;", "const float denom = G;", NVFP4_PINS),
    ("nvfp4 FFN: gate and up swapped",
     "float g = gu[n], u = gu[F + n];", "float g = gu[F + n], u = gu[n];", NVFP4_PINS),
    ("nvfp4 FFN: h quantised with the activation global",
     "orc_nvfp4_quantize(h, 1, F, Gh, hc, hs);", "orc_nvfp4_quantize(h, 1, F, Gx, hc, hs);", NVFP4_PINS),
    ("int4 FFN: up rows read the gate rows' scales",
     "gu_scale[ru * Gh + i / 64]", "gu_scale[rg * Gh + i / 64]", METHOD_PINS),
    ("int4 FFN: SiLU on the up projection",
     "u += wu * xf[i];\n    }\n    h[n] = g / (1.0f + expf(-g)) * u;",
     "u += wu * xf[i];\n    }\n    h[n] = u / (1.0f + expf(-u)) * g;", METHOD_PINS),
    ("int4 FFN: down weights transposed",
     "orc_dequant_one(d_codes[(size_t)c * F + n]", "orc_dequant_one(d_codes[(size_t)n * H + c]", METHOD_PINS),
    ("route: ties go to the higher expert id",
     "if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] >= l[best]) best = e;", METHOD_PINS),
    ("route: weights not renormalised over the selected experts",
     "w[(size_t)t * k + j] = p[idx[(size_t)t * k + j]] / Ssel;",
     "w[(size_t)t * k + j] = p[idx[(size_t)t * k + j]] / S;", METHOD_PINS),
    ("permute: rows of an expert in reverse order",
     "int pos = offsets[e] + fill[e]++;", "int pos = offsets[e] + counts[e] - 1 - fill[e]++;", METHOD_PINS),
    ("quantiser: min rounded to nearest instead of toward -inf",
     "uint16_t mh = orc_f32_to_f16(mn, 1);", "uint16_t mh = orc_f32_to_f16(mn, 0);", METHOD_PINS),
    ("dequant: scale and min swapped",
     "fmaf((float)q, orc_f16_to_f32(s), orc_f16_to_f32(m))",
     "fmaf((float)q, orc_f16_to_f32(m), orc_f16_to_f32(s))", METHOD_PINS),
    ("clip search: ratios 1.0 down to 0.62 instead of 0.81",
     "return (float)(100 - i) / 100.0f;", "return (float)(100 - 2 * i) / 100.0f;", CLIP_PINS),
    ("clip search: asymmetric min rounded to nearest",
     "uint16_t mh = orc_f32_to_f16(p * mn, 1);", "uint16_t mh = orc_f32_to_f16(p * mn, 0);", CLIP_PINS),
    ("clip search: absolute instead of squared error",
     "float d = (qi - 8.0f) * s - wg[i];\n          err += d * d;",
     "float d = (qi - 8.0f) * s - wg[i];\n          err += fabsf(d);", CLIP_PINS),
    ("clip search: the largest error wins",
     "          q[i] = (uint8_t)qi;\n          float d = fmaf(qi, s, m) - wg[i];\n          err += d * d;\n        }\n"
     "        if (err < best) {",
     "          q[i] = (uint8_t)qi;\n          float d = fmaf(qi, s, m) - wg[i];\n          err += d * d;\n        }\n"
     "        if (-err < best) {", CLIP_PINS),
    ("symmetric group 128: zero point 7",
     "qi = nearbyintf(wg[i] / s) + 8.0f;", "qi = nearbyintf(wg[i] / s) + 7.0f;", CLIP_PINS),
    ("symmetric group 128: scale amax / 7.5 dropped to amax / 8",
     "uint16_t sh = orc_f32_to_f16(t / 15.0f, 0);", "uint16_t sh = orc_f32_to_f16(t / 16.0f, 0);", CLIP_PINS),
    ("symmetric group 128: dequant with zero point 7",
     "return ((float)q - 8.0f) * orc_f16_to_f32(s);", "return ((float)q - 7.0f) * orc_f16_to_f32(s);", CLIP_PINS),
    ("symmetric group 128 FFN: down scales indexed by output row only",
     "d_scale[(size_t)c * Gf + n / 128]", "d_scale[(size_t)c * Gf]", CLIP_PINS),
    ("router linear: weight matrix transposed",
     "orc_bf16_to_f32(wr[(size_t)e * H + i])", "orc_bf16_to_f32(wr[(size_t)i * E + e])", ROUTER_PINS),
    ("router linear: first channel skipped",
     "      for (int i = 0; i < H; ++i)\n        acc += orc_bf16_to_f32(x[(size_t)t * H + i])",
     "      for (int i = 1; i < H; ++i)\n        acc += orc_bf16_to_f32(x[(size_t)t * H + i])", ROUTER_PINS),
    ("shared expert: weight one half instead of one",
     "w1[(size_t)t * k1 + k] = 1.0f;", "w1[(size_t)t * k1 + k] = 0.5f;", SHARED_PINS),
    ("shared expert: applied to the wrong token",
     "    orc_expert_ffn_w4(x + (size_t)t * H, H, F, s_gu_codes,",
     "    orc_expert_ffn_w4(x + (size_t)((t + 1) % T) * H, H, F, s_gu_codes,", SHARED_PINS),
    ("combine: routing weight dropped",
     "acc += w[(size_t)t * k + j] * Yrows[((size_t)t * k + j) * H + c];",
     "acc += Yrows[((size_t)t * k + j) * H + c];", METHOD_PINS),
]


@pytest.mark.parametrize("name,old,new,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_fail_on_planted_mistake(name, old, new, pins, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    bad = tmp_path / "moe_oracle_mutant.c"
    bad.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(bad), "-lm"])
    # no conftest in the child: the pin files need neither torch nor a GPU
    env = dict(os.environ, ORACLE_LIB=str(so), PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "--noconftest",
                        pins],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, (f"pins in {pins} did not catch: {name}\n"
                               + r.stdout[-2000:] + r.stderr[-2000:])
