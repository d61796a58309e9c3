/*
 * moe_oracle.c -- plain, slow CPU oracle for the routed 4-bit MoE FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or helper with the CUDA
 * path: every number format below is decoded from its definition here.
 *
 * What it computes, and where the pages define it:
 *   - int4 asymmetric group-64 experts, f16 scale + f16 min per group
 *     ("Drama 3 int4 (drama-rs format)", section "What's quantized", table row
 *     for routed MoE experts); the affine map w = q*scale + min is the MLX
 *     "packed affine" form the same weights map to losslessly ("drama-rs",
 *     section "Apple Silicon (MLX)"; "DRAMA-3 MLX expert-only 4-bit",
 *     section "Quantization and provenance").
 *   - 256 routed experts, 3 projections each ("Drama 3 - NVFP4 routed
 *     experts", section "Quantization", first bullet); the expert MLP of the
 *     Qwen3.5-MoE backbone is a SwiGLU FFN (gate, up, down) ("drama-rs",
 *     first bullet list).
 *   - softmax routing with renormalised top-k over the router logits, and the
 *     router-weighted combine (the router is bf16 per "Drama 3 int4",
 *     "What's quantized"; top-k = 8, renormalisation and the lowest-index tie
 *     break are the readings taken where the pages are silent).
 *   - NVFP4 experts: packed E2M1 codes, one E4M3 scale per 16 input channels,
 *     one FP32 global scale per matrix, gate and up sharing it, dynamic
 *     per-token activation scales ("Drama 3 - NVFP4 routed experts",
 *     section "Quantization", bullets 2 and 4).
 *   - the MSE clip search over 20 clipping ratios 1.00 -> 0.81 ("Drama 3 int4
 *     (drama-rs format)", "What's quantized"; "drama-3-w4a16", "How it was
 *     made") for the asymmetric group-64 format and for the symmetric
 *     group-128 format with zero point 8 ("drama-3-w4a16", "At a glance").
 *   - the bf16 router linear (logits = Wr x) and a shared expert beside the
 *     routed ones ("Drama 3 int4 (drama-rs format)", "What's quantized";
 *     "Drama 3 - NVFP4 routed experts", "Quantization").
 *
 * Precision: the FFN accumulates in fp32 with k ascending, dequantises with
 * one fp32 fused multiply-add (q*s + m, single rounding), and rounds the
 * combined output to bf16 with round-to-nearest-even.  Build with
 * -ffp-contract=off so the compiler fuses nothing the source does not.
 *
 * Parity status of every function is stated beside it; all are pinned by the
 * CPU tests (closed forms, brute force, library cross-checks, invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16, decoded and encoded from the format definition         */
/* (1 sign bit, 5 exponent bits with bias 15, 10 mantissa bits).             */
/* ------------------------------------------------------------------------ */

ORC_API float orc_f16_to_f32(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(m | 1024), e - 25);
  return (float)(s ? -v : v);
}

/* mode: 0 = nearest-even, 1 = toward -inf, 2 = toward +inf */
ORC_API uint16_t orc_f32_to_f16(float x, int mode) {
  if (isnan(x)) return 0x7E00;
  int neg = signbit(x) ? 1 : 0;
  double a = fabs((double)x);
  /* magnitude rounding: 0 nearest-even, 1 away from zero, 2 toward zero */
  int mag = 0;
  if (mode == 1) mag = neg ? 1 : 2;
  if (mode == 2) mag = neg ? 2 : 1;
  uint16_t sign = (uint16_t)(neg << 15);
  if (isinf(a)) return (uint16_t)(sign | (mag == 2 ? 0x7BFF : 0x7C00));
  double q; /* quantum (spacing of binary16 values around a) */
  if (a < ldexp(1.0, -14)) {
    q = ldexp(1.0, -24);
  } else {
    int ex;
    frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) */
    q = ldexp(1.0, (ex - 1) - 10);
  }
  double n = a / q; /* exact: a has 24 significant bits, q is a power of two */
  double fl = floor(n), r;
  if (mag == 1) r = ceil(n);
  else if (mag == 2) r = fl;
  else {
    double frac = n - fl;
    if (frac > 0.5) r = fl + 1.0;
    else if (frac < 0.5) r = fl;
    else r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  }
  double v = r * q;
  if (v > 65504.0) return (uint16_t)(sign | (mag == 2 ? 0x7BFF : 0x7C00));
  if (v < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(v / ldexp(1.0, -24)));
  int ex;
  frexp(v, &ex);
  int E = ex - 1;
  uint16_t mant = (uint16_t)(v / ldexp(1.0, E - 10) - 1024.0);
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | mant);
}

/* ------------------------------------------------------------------------ */
/* bfloat16: the upper 16 bits of a binary32; rounding to nearest-even on    */
/* the dropped 16 bits.                                                      */
/* ------------------------------------------------------------------------ */

ORC_API float orc_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

ORC_API uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t lower = u & 0xFFFFu, upper = u >> 16;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
  return (uint16_t)upper;
}

/* ------------------------------------------------------------------------ */
/* FP4 E2M1 and FP8 E4M3 (the OCP "FN" variant: no infinities, S.1111.111    */
/* is NaN, largest finite 448), decoded and encoded from their definitions.  */
/* ------------------------------------------------------------------------ */

ORC_API float orc_e2m1_to_f32(uint8_t c) {
  int e = (c >> 1) & 3, m = c & 1;
  float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
  return (c & 8) ? -mag : mag;
}

/* round to nearest, ties to the even code, saturating at +-6; sign kept */
ORC_API uint8_t orc_f32_to_e2m1(float v) {
  uint8_t sign = signbit(v) ? 8 : 0;
  float a = fabsf(v);
  if (isnan(a)) return (uint8_t)(sign | 7);
  uint8_t best = 0;
  for (uint8_t c = 1; c < 8; ++c) {
    float dc = fabsf(orc_e2m1_to_f32(c) - a), db = fabsf(orc_e2m1_to_f32(best) - a);
    if (dc < db || (dc == db && (c & 1) == 0)) best = c;
  }
  if (a >= 6.0f) best = 7;
  return (uint8_t)(sign | best);
}

ORC_API float orc_e4m3_to_f32(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  float v;
  if (e == 15 && m == 7) v = NAN;
  else if (e == 0) v = ldexpf((float)m / 8.0f, -6);
  else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -v : v;
}

/* round to nearest-even, saturating to +-448 (never produces NaN from a
 * finite input) */
ORC_API uint8_t orc_f32_to_e4m3(float v) {
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double a = fabs((double)v);
  if (isnan(v)) return (uint8_t)(sign | 0x7F);
  double q;
  if (a < ldexp(1.0, -6)) q = ldexp(1.0, -9);
  else {
    int ex;
    frexp(a, &ex);
    q = ldexp(1.0, (ex - 1) - 3);
  }
  double n = a / q, fl = floor(n), r, frac = n - fl;
  if (frac > 0.5) r = fl + 1.0;
  else if (frac < 0.5) r = fl;
  else r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  double mag = r * q;
  if (mag > 448.0) mag = 448.0;
  if (mag < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(mag / ldexp(1.0, -9)));
  int ex;
  frexp(mag, &ex);
  int E = ex - 1;
  uint8_t mant = (uint8_t)(mag / ldexp(1.0, E - 3) - 8.0);
  return (uint8_t)(sign | (uint8_t)((E + 7) << 3) | mant);
}

/* ------------------------------------------------------------------------ */
/* int4 asymmetric group-64 quantizer (test-data generator).                 */
/* For each row and each group of 64 consecutive input channels:             */
/*   mn, mx = group min, max;                                                */
/*   m = f16(mn) rounded toward -inf;                                        */
/*   s = f16((mx - m) / 15) rounded toward +inf;                             */
/*   q = clamp(round-half-even((w - m) / s), 0, 15), all in fp32;            */
/*   s == 0 (a constant group) gives q = 0.                                  */
/* The directed roundings make [m, m + 15 s] cover [mn, mx], so no code      */
/* clips.  Groups run along the input (K) dimension.                         */
/* Parity: pinned (error bound, coverage, closed-form groups).               */
/* ------------------------------------------------------------------------ */

ORC_API void orc_quantize_w4(const float *w, int N, int K, uint8_t *codes,
                             uint16_t *scale, uint16_t *minv) {
  const int G = K / 64;
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const float *wg = w + (size_t)n * K + (size_t)g * 64;
      float mn = wg[0], mx = wg[0];
      for (int i = 1; i < 64; ++i) {
        if (wg[i] < mn) mn = wg[i];
        if (wg[i] > mx) mx = wg[i];
      }
      uint16_t mh = orc_f32_to_f16(mn, 1);
      float m = orc_f16_to_f32(mh);
      float span = mx - m;
      uint16_t sh = orc_f32_to_f16(span / 15.0f, 2);
      float s = orc_f16_to_f32(sh);
      scale[(size_t)n * G + g] = sh;
      minv[(size_t)n * G + g] = mh;
      for (int i = 0; i < 64; ++i) {
        float q = 0.0f;
        if (s > 0.0f) {
          float t = (wg[i] - m) / s;
          q = nearbyintf(t);
          if (q < 0.0f) q = 0.0f;
          if (q > 15.0f) q = 15.0f;
        }
        codes[(size_t)n * K + (size_t)g * 64 + i] = (uint8_t)q;
      }
    }
  }
}

/* Canonical packing: eight codes per little-endian 32-bit word along K,
 * element k in bits 4*(k mod 8) of word k/8 (lower channel in the lower
 * nibble).  Parity: pinned by the round trip. */
ORC_API void orc_pack_nibbles(const uint8_t *codes, int N, int K, uint32_t *words) {
  for (int n = 0; n < N; ++n)
    for (int k8 = 0; k8 < K / 8; ++k8) {
      uint32_t wd = 0;
      for (int i = 0; i < 8; ++i)
        wd |= (uint32_t)(codes[(size_t)n * K + (size_t)k8 * 8 + i] & 15u) << (4 * i);
      words[(size_t)n * (K / 8) + k8] = wd;
    }
}

ORC_API void orc_unpack_nibbles(const uint32_t *words, int N, int K, uint8_t *codes) {
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      codes[(size_t)n * K + k] =
          (uint8_t)((words[(size_t)n * (K / 8) + k / 8] >> (4 * (k % 8))) & 15u);
}

/* Dequantised weight: one fp32 fused multiply-add, q*s + m.
 * Parity: pinned (hand-set values). */
ORC_API float orc_dequant_one(uint8_t q, uint16_t s, uint16_t m) {
  return fmaf((float)q, orc_f16_to_f32(s), orc_f16_to_f32(m));
}

ORC_API void orc_dequant_w4(const uint8_t *codes, const uint16_t *scale,
                            const uint16_t *minv, int N, int K, float *out) {
  const int G = K / 64;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      out[(size_t)n * K + k] = orc_dequant_one(codes[(size_t)n * K + k],
                                               scale[(size_t)n * G + k / 64],
                                               minv[(size_t)n * G + k / 64]);
}

/* ------------------------------------------------------------------------ */
/* Routing.  Experts ordered by logit, larger first, equal logits to the     */
/* lower index first; the first k are selected (idx in that order).          */
/* p = softmax over all E logits (max-subtracted, fp32 exp); the routing     */
/* weights are the selected p renormalised to sum to one.                    */
/* Parity: pinned (brute-force sort, k = 1, k = E, softmax-of-selected       */
/* identity, hand-set ties).                                                 */
/* ------------------------------------------------------------------------ */

ORC_API void orc_route(const float *logits, int T, int E, int k, int32_t *idx, float *w) {
  float *p = (float *)malloc(sizeof(float) * (size_t)E);
  unsigned char *taken = (unsigned char *)malloc((size_t)E);
  for (int t = 0; t < T; ++t) {
    const float *l = logits + (size_t)t * E;
    float M = l[0];
    for (int e = 1; e < E; ++e)
      if (l[e] > M) M = l[e];
    float S = 0.0f;
    for (int e = 0; e < E; ++e) {
      p[e] = expf(l[e] - M);
      S += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] = p[e] / S;
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e; /* strict: ties keep lower e */
      }
      taken[best] = 1;
      idx[(size_t)t * k + j] = best;
    }
    float Ssel = 0.0f;
    for (int j = 0; j < k; ++j) Ssel += p[idx[(size_t)t * k + j]];
    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = p[idx[(size_t)t * k + j]] / Ssel;
  }
  free(p);
  free(taken);
}

/* ------------------------------------------------------------------------ */
/* Permutation: rows r = t*k + j grouped by expert.                          */
/*   counts[e]  = number of rows routed to e                                 */
/*   offsets    = exclusive scan of counts, offsets[E] = T*k                 */
/*   sorted_rows lists r ordered by (expert, r) ascending                    */
/*   inv[r]     = position of r in sorted_rows                               */
/* Parity: pinned (brute-force stable sort, invariants).                     */
/* ------------------------------------------------------------------------ */

ORC_API void orc_permute(const int32_t *idx, int T, int k, int E, int32_t *counts,
                         int32_t *offsets, int32_t *sorted_rows, int32_t *inv) {
  const int R = T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int r = 0; r < R; ++r) counts[idx[r]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
  for (int r = 0; r < R; ++r) {
    int e = idx[r];
    int pos = offsets[e] + fill[e]++;
    sorted_rows[pos] = r;
    inv[r] = pos;
  }
  free(fill);
}

/* ------------------------------------------------------------------------ */
/* One expert's SwiGLU FFN on one bf16 activation row, dequantising every    */
/* weight literally inside the dot products.                                 */
/*   gate_up: [2F][H] codes, rows [0, F) gate, rows [F, 2F) up               */
/*   down:    [H][F] codes                                                   */
/*   g_n = sum_k w_g[n][k] x[k];  u_n likewise;  (fp32, k ascending)         */
/*   h_n = g_n / (1 + exp(-g_n)) * u_n                                       */
/*   Y_c = sum_n w_d[c][n] h_n                                               */
/* h_out (optional) receives h.  Parity: pinned (constant-code and           */
/* permutation-code closed forms; library cross-check).                      */
/* ------------------------------------------------------------------------ */

ORC_API void orc_expert_ffn_w4(const uint16_t *x, int H, int F,
                               const uint8_t *gu_codes, const uint16_t *gu_scale,
                               const uint16_t *gu_min, const uint8_t *d_codes,
                               const uint16_t *d_scale, const uint16_t *d_min,
                               float *Y, float *h_out) {
  const int Gh = H / 64, Gf = F / 64;
  float *xf = (float *)malloc(sizeof(float) * (size_t)H);
  float *h = (float *)malloc(sizeof(float) * (size_t)F);
  for (int i = 0; i < H; ++i) xf[i] = orc_bf16_to_f32(x[i]);
  for (int n = 0; n < F; ++n) {
    float g = 0.0f, u = 0.0f;
    for (int i = 0; i < H; ++i) {
      size_t rg = (size_t)n, ru = (size_t)(F + n);
      float wg = orc_dequant_one(gu_codes[rg * H + i], gu_scale[rg * Gh + i / 64],
                                 gu_min[rg * Gh + i / 64]);
      float wu = orc_dequant_one(gu_codes[ru * H + i], gu_scale[ru * Gh + i / 64],
                                 gu_min[ru * Gh + i / 64]);
      g += wg * xf[i];
      u += wu * xf[i];
    }
    h[n] = g / (1.0f + expf(-g)) * u;
  }
  for (int c = 0; c < H; ++c) {
    float acc = 0.0f;
    for (int n = 0; n < F; ++n) {
      float wd = orc_dequant_one(d_codes[(size_t)c * F + n], d_scale[(size_t)c * Gf + n / 64],
                                 d_min[(size_t)c * Gf + n / 64]);
      acc += wd * h[n];
    }
    Y[c] = acc;
  }
  if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)F);
  free(xf);
  free(h);
}

/* Router-weighted combine: y[t] = sum_{j ascending} w[t][j] * Yrows[t*k+j],
 * fp32, then round-to-nearest-even to bf16.  Parity: pinned (one-hot
 * weights, dense-vs-sparse identity). */
ORC_API void orc_combine(const float *Yrows, const float *w, int T, int k, int H, uint16_t *y) {
  for (int t = 0; t < T; ++t)
    for (int c = 0; c < H; ++c) {
      float acc = 0.0f;
      for (int j = 0; j < k; ++j)
        acc += w[(size_t)t * k + j] * Yrows[((size_t)t * k + j) * H + c];
      y[(size_t)t * H + c] = orc_f32_to_bf16(acc);
    }
}

/* Shared expert: one more SwiGLU expert applied to every token, added after
 * the routed experts with weight 1:
 *   y_t = bf16( (sum over j < k, in order, of w[t][j] Y_(t,j))  +  1 * Y_s(x_t) )
 * -- the combine of k + 1 rows whose last row is the shared expert's, with
 * weight 1.  The pages list a shared expert beside the routed ones ("Drama 3
 * int4 (drama-rs format)", table "What's quantized"; "Drama 3 - NVFP4 routed
 * experts", section "Quantization"); weight 1, its place after the routed
 * sum, and its int4 storage (in the routed experts' format) are the reading
 * taken here.  idx/w receive the k routed choices; y_rows (optional) [T][k+1][H]
 * the rows.  Parity: pinned (zero shared weights give the routed-only result;
 * zero routed weights give the shared expert alone; the composition of the
 * pinned FFN and combine). */
ORC_API void orc_moe_forward_w4_shared(const uint16_t *x, const float *logits, int T, int E, int k,
                                       int H, int F, const uint8_t *const *gu_codes,
                                       const uint16_t *const *gu_scale,
                                       const uint16_t *const *gu_min,
                                       const uint8_t *const *d_codes,
                                       const uint16_t *const *d_scale,
                                       const uint16_t *const *d_min, const uint8_t *s_gu_codes,
                                       const uint16_t *s_gu_scale, const uint16_t *s_gu_min,
                                       const uint8_t *s_d_codes, const uint16_t *s_d_scale,
                                       const uint16_t *s_d_min, int32_t *idx, float *w,
                                       float *y_rows, uint16_t *y) {
  const int k1 = k + 1;
  orc_route(logits, T, E, k, idx, w);
  float *rows = y_rows ? y_rows : (float *)malloc(sizeof(float) * (size_t)T * k1 * H);
  float *w1 = (float *)malloc(sizeof(float) * (size_t)T * k1);
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      orc_expert_ffn_w4(x + (size_t)t * H, H, F, gu_codes[e], gu_scale[e], gu_min[e], d_codes[e],
                        d_scale[e], d_min[e], rows + ((size_t)t * k1 + j) * H, NULL);
      w1[(size_t)t * k1 + j] = w[(size_t)t * k + j];
    }
    orc_expert_ffn_w4(x + (size_t)t * H, H, F, s_gu_codes, s_gu_scale, s_gu_min, s_d_codes,
                      s_d_scale, s_d_min, rows + ((size_t)t * k1 + k) * H, NULL);
    w1[(size_t)t * k1 + k] = 1.0f;
  }
  orc_combine(rows, w1, T, k1, H, y);
  free(w1);
  if (!y_rows) free(rows);
}

/* ------------------------------------------------------------------------ */
/* Router linear: logits[t][e] = sum_k x[t][k] * Wr[e][k], x and Wr bf16,    */
/* each product and the running sum fp32, k ascending; no bias.  The router  */
/* keeps bf16 weights ("Drama 3 int4 (drama-rs format)", table "What's       */
/* quantized": embeddings, router, norms bf16 / f32; "DRAMA-3 MLX            */
/* expert-only 4-bit", section "Quantization and provenance": routers retain */
/* source BF16); fp32 accumulation and no bias are the reading taken here.  */
/* Parity: pinned (one-hot rows select a channel of x exactly; a float64     */
/* matmul within the fp32 summation bound; linearity in x).                  */
/* ------------------------------------------------------------------------ */

ORC_API void orc_router_logits(const uint16_t *x, const uint16_t *wr, int T, int E, int H,
                               float *logits) {
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      float acc = 0.0f;
      for (int i = 0; i < H; ++i)
        acc += orc_bf16_to_f32(x[(size_t)t * H + i]) * orc_bf16_to_f32(wr[(size_t)e * H + i]);
      logits[(size_t)t * E + e] = acc;
    }
}

/* Whole routed MoE FFN for T tokens: route, then for every (t, j) the
 * expert FFN of expert idx[t][j] on x[t], then the combine.  Expert weights
 * come as per-expert pointer tables (an entry may be NULL when the expert is
 * never selected).  y_rows (optional) receives the per-row fp32 outputs. */
ORC_API void orc_moe_forward_w4(const uint16_t *x, const float *logits, int T, int E, int k,
                                int H, int F, const uint8_t *const *gu_codes,
                                const uint16_t *const *gu_scale, const uint16_t *const *gu_min,
                                const uint8_t *const *d_codes, const uint16_t *const *d_scale,
                                const uint16_t *const *d_min, int32_t *idx, float *w,
                                float *y_rows, uint16_t *y) {
  orc_route(logits, T, E, k, idx, w);
  float *rows = y_rows ? y_rows : (float *)malloc(sizeof(float) * (size_t)T * k * H);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      orc_expert_ffn_w4(x + (size_t)t * H, H, F, gu_codes[e], gu_scale[e], gu_min[e],
                        d_codes[e], d_scale[e], d_min[e], rows + ((size_t)t * k + j) * H, NULL);
    }
  orc_combine(rows, w, T, k, H, y);
  if (!y_rows) free(rows);
}

/* ------------------------------------------------------------------------ */
/* MSE clip search, and the symmetric group-128 int4 format.                 */
/*                                                                           */
/* "Drama 3 int4 (drama-rs format)", table "What's quantized": routed        */
/* experts int4, asymmetric, group 64, f16 scale + min, MSE clip search.     */
/* "drama-3-w4a16", section "How it was made": round-to-nearest int4, one    */
/* scale per 128 input weights, each scale chosen from 20 clipping ratios    */
/* (1.0 down to 0.81) by minimum squared error; table "At a glance": int4,   */
/* symmetric, group 128, GPTQ packing.                                       */
/* Readings (the pages give no formulas):                                    */
/*   - ratio i = 0..19 is p_i = (100 - i) / 100 (one fp32 division); the     */
/*     candidate range is the group's range scaled by p_i;                   */
/*   - the squared error of a candidate is summed in fp32 over the group's   */
/*     channels in ascending order, each term d * d with d the dequantised   */
/*     value minus the weight; the smallest error wins, ties to the larger   */
/*     ratio (smaller i);                                                    */
/*   - asymmetric (group 64): m = f16(p mn) toward -inf, s = f16((p mx - m)  */
/*     / 15) toward +inf, codes as in orc_quantize_w4; p = 1 is exactly      */
/*     orc_quantize_w4's choice;                                             */
/*   - symmetric (group 128), with GPTQ's zero point 8: w = (q - 8) s,       */
/*     q in 0..15, s = f16(2 p amax / 15) nearest-even (fp32 p * amax, then  */
/*     * 2, then / 15), q = clamp(rint(w / s) + 8, 0, 15); s = 0 gives q = 8.*/
/* Parity: pinned (p = 1 equals the plain quantiser; the chosen candidate's  */
/* error is the brute-force minimum over the 20; error bound of unclipped   */
/* elements; the mean relative error on Gaussian weights the w4a16 page      */
/* reports for int4 group 128).                                              */
/* ------------------------------------------------------------------------ */

static float clip_ratio(int i) { return (float)(100 - i) / 100.0f; }

ORC_API void orc_quantize_w4_clip(const float *w, int N, int K, uint8_t *codes,
                                  uint16_t *scale, uint16_t *minv) {
  const int G = K / 64;
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const float *wg = w + (size_t)n * K + (size_t)g * 64;
      float mn = wg[0], mx = wg[0];
      for (int i = 1; i < 64; ++i) {
        if (wg[i] < mn) mn = wg[i];
        if (wg[i] > mx) mx = wg[i];
      }
      float best = INFINITY;
      for (int c = 0; c < 20; ++c) {
        const float p = clip_ratio(c);
        uint16_t mh = orc_f32_to_f16(p * mn, 1);
        float m = orc_f16_to_f32(mh);
        float span = p * mx - m;
        uint16_t sh = orc_f32_to_f16(span / 15.0f, 2);
        float s = orc_f16_to_f32(sh);
        uint8_t q[64];
        float err = 0.0f;
        for (int i = 0; i < 64; ++i) {
          float qi = 0.0f;
          if (s > 0.0f) {
            qi = nearbyintf((wg[i] - m) / s);
            if (qi < 0.0f) qi = 0.0f;
            if (qi > 15.0f) qi = 15.0f;
          }
          q[i] = (uint8_t)qi;
          float d = fmaf(qi, s, m) - wg[i];
          err += d * d;
        }
        if (err < best) {
          best = err;
          scale[(size_t)n * G + g] = sh;
          minv[(size_t)n * G + g] = mh;
          memcpy(codes + (size_t)n * K + (size_t)g * 64, q, 64);
        }
      }
    }
  }
}

ORC_API void orc_quantize_sym128(const float *w, int N, int K, uint8_t *codes, uint16_t *scale) {
  const int G = K / 128;
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const float *wg = w + (size_t)n * K + (size_t)g * 128;
      float amax = 0.0f;
      for (int i = 0; i < 128; ++i) {
        float a = fabsf(wg[i]);
        if (a > amax) amax = a;
      }
      float best = INFINITY;
      for (int c = 0; c < 20; ++c) {
        const float p = clip_ratio(c);
        float t = p * amax;
        t = 2.0f * t;
        uint16_t sh = orc_f32_to_f16(t / 15.0f, 0);
        float s = orc_f16_to_f32(sh);
        uint8_t q[128];
        float err = 0.0f;
        for (int i = 0; i < 128; ++i) {
          float qi = 8.0f;
          if (s > 0.0f) {
            qi = nearbyintf(wg[i] / s) + 8.0f;
            if (qi < 0.0f) qi = 0.0f;
            if (qi > 15.0f) qi = 15.0f;
          }
          q[i] = (uint8_t)qi;
          float d = (qi - 8.0f) * s - wg[i];
          err += d * d;
        }
        if (err < best) {
          best = err;
          scale[(size_t)n * G + g] = sh;
          memcpy(codes + (size_t)n * K + (size_t)g * 128, q, 128);
        }
      }
    }
  }
}

/* w = (q - 8) * s, exact in fp32 (s has 11 significant bits, q - 8 four). */
ORC_API float orc_dequant_sym128(uint8_t q, uint16_t s) {
  return ((float)q - 8.0f) * orc_f16_to_f32(s);
}

/* One expert's SwiGLU FFN on one bf16 row with symmetric group-128 weights,
 * each weight dequantised literally by orc_dequant_sym128; otherwise as
 * orc_expert_ffn_w4 (fp32 sums in ascending order, h = SiLU(g) * u). */
ORC_API void orc_expert_ffn_sym128(const uint16_t *x, int H, int F, const uint8_t *gu_codes,
                                   const uint16_t *gu_scale, const uint8_t *d_codes,
                                   const uint16_t *d_scale, float *Y, float *h_out) {
  const int Gh = H / 128, Gf = F / 128;
  float *xf = (float *)malloc(sizeof(float) * (size_t)H);
  float *h = (float *)malloc(sizeof(float) * (size_t)F);
  for (int i = 0; i < H; ++i) xf[i] = orc_bf16_to_f32(x[i]);
  for (int n = 0; n < F; ++n) {
    float g = 0.0f, u = 0.0f;
    for (int i = 0; i < H; ++i) {
      size_t rg = (size_t)n, ru = (size_t)(F + n);
      g += orc_dequant_sym128(gu_codes[rg * H + i], gu_scale[rg * Gh + i / 128]) * xf[i];
      u += orc_dequant_sym128(gu_codes[ru * H + i], gu_scale[ru * Gh + i / 128]) * xf[i];
    }
    h[n] = g / (1.0f + expf(-g)) * u;
  }
  for (int c = 0; c < H; ++c) {
    float acc = 0.0f;
    for (int n = 0; n < F; ++n)
      acc += orc_dequant_sym128(d_codes[(size_t)c * F + n], d_scale[(size_t)c * Gf + n / 128]) * h[n];
    Y[c] = acc;
  }
  if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)F);
  free(xf);
  free(h);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 (E2M1 codes, E4M3 scale per 16 input channels, FP32 global scale).  */
/* Global scale of a tensor (a weight matrix, gate and up taken together, or */
/* one activation row): G = amax / (448 * 6); G = 1 when amax == 0.          */
/* Block scale: S_b = E4M3(amax_b / (6 G)), saturating; codes               */
/* E2M1(v / (S_b G)), saturating; a zero S_b gives zero codes.               */
/* ("Drama 3 - NVFP4 routed experts", section "Quantization": round-to-      */
/* nearest, one E4M3 scale per 16 input weights, FP32 global per matrix,     */
/* dynamic per-token FP32 activation scales with E4M3 block scales.)         */
/* Parity: pinned.  Decode tables exhaustively; the global by hand values;  */
/* the quantiser by round trip, per-(row, block) scales and error bound; the */
/* GEMV by a constant-code closed form, one-hot rows with a distinct scale   */
/* per (row, block), and a float64 matmul of the decoded operands within the */
/* fp32 summation bound; the FFN by a constant-code closed form and a        */
/* stage-wise composition of the pinned pieces.                              */
/* ------------------------------------------------------------------------ */

ORC_API float orc_nvfp4_global(const float *v, size_t n) {
  float amax = 0.0f;
  for (size_t i = 0; i < n; ++i) {
    float a = fabsf(v[i]);
    if (a > amax) amax = a;
  }
  if (amax == 0.0f) return 1.0f;
  return amax / 2688.0f;
}

/* Quantise rows [N][K] (K % 16 == 0) with a given global scale G. */
ORC_API void orc_nvfp4_quantize(const float *v, int N, int K, float G, uint8_t *codes,
                                uint8_t *sf) {
  const float denom = 6.0f * G;
  for (int n = 0; n < N; ++n)
    for (int b = 0; b < K / 16; ++b) {
      const float *vb = v + (size_t)n * K + (size_t)b * 16;
      float amax = 0.0f;
      for (int i = 0; i < 16; ++i) {
        float a = fabsf(vb[i]);
        if (a > amax) amax = a;
      }
      uint8_t s8 = orc_f32_to_e4m3(amax / denom);
      float sb = orc_e4m3_to_f32(s8);
      sf[(size_t)n * (K / 16) + b] = s8;
      float scale = sb * G;
      for (int i = 0; i < 16; ++i)
        codes[(size_t)n * K + (size_t)b * 16 + i] =
            (sb == 0.0f) ? (uint8_t)0 : orc_f32_to_e2m1(vb[i] / scale);
    }
}

/* y[n] = (sum_k dec(a_k) sa_b * dec(w[n][k]) sw_b) * Ga * Gw, fp32 literal. */
ORC_API void orc_nvfp4_gemv(const uint8_t *a_codes, const uint8_t *a_sf, float Ga,
                            const uint8_t *w_codes, const uint8_t *w_sf, float Gw, int N, int K,
                            float *y) {
  for (int n = 0; n < N; ++n) {
    float acc = 0.0f;
    for (int k = 0; k < K; ++k) {
      float a = orc_e2m1_to_f32(a_codes[k]) * orc_e4m3_to_f32(a_sf[k / 16]);
      float wv = orc_e2m1_to_f32(w_codes[(size_t)n * K + k]) *
                 orc_e4m3_to_f32(w_sf[(size_t)n * (K / 16) + k / 16]);
      acc += a * wv;
    }
    y[n] = acc * (Ga * Gw);
  }
}

/* One expert's NVFP4 SwiGLU FFN on one bf16 row: x is quantised per token,
 * h is re-quantised per row before the down projection.
 *   gu: [2F][H] codes + [2F][H/16] scales, shared global G_gu
 *   d:  [H][F] codes + [H][F/16] scales, global G_d
 * h_codes/h_sf/h_G (optional) receive the quantised h. */
ORC_API void orc_expert_ffn_nvfp4(const uint16_t *x, int H, int F, const uint8_t *gu_codes,
                                  const uint8_t *gu_sf, float G_gu, const uint8_t *d_codes,
                                  const uint8_t *d_sf, float G_d, float *Y, float *h_out,
                                  uint8_t *h_codes, uint8_t *h_sf, float *h_G) {
  float *xf = (float *)malloc(sizeof(float) * (size_t)H);
  uint8_t *xc = (uint8_t *)malloc((size_t)H), *xs = (uint8_t *)malloc((size_t)H / 16);
  float *gu = (float *)malloc(sizeof(float) * 2 * (size_t)F);
  float *h = (float *)malloc(sizeof(float) * (size_t)F);
  uint8_t *hc = (uint8_t *)malloc((size_t)F), *hs = (uint8_t *)malloc((size_t)F / 16);
  for (int i = 0; i < H; ++i) xf[i] = orc_bf16_to_f32(x[i]);
  float Gx = orc_nvfp4_global(xf, (size_t)H);
  orc_nvfp4_quantize(xf, 1, H, Gx, xc, xs);
  orc_nvfp4_gemv(xc, xs, Gx, gu_codes, gu_sf, G_gu, 2 * F, H, gu);
  for (int n = 0; n < F; ++n) {
    float g = gu[n], u = gu[F + n];
    h[n] = g / (1.0f + expf(-g)) * u;
  }
  float Gh = orc_nvfp4_global(h, (size_t)F);
  orc_nvfp4_quantize(h, 1, F, Gh, hc, hs);
  orc_nvfp4_gemv(hc, hs, Gh, d_codes, d_sf, G_d, H, F, Y);
  if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)F);
  if (h_codes) memcpy(h_codes, hc, (size_t)F);
  if (h_sf) memcpy(h_sf, hs, (size_t)F / 16);
  if (h_G) *h_G = Gh;
  free(xf); free(xc); free(xs); free(gu); free(h); free(hc); free(hs);
}

/* The down projection alone from given quantised h (stage-wise check). */
ORC_API void orc_down_nvfp4(const uint8_t *h_codes, const uint8_t *h_sf, float Gh, int H, int F,
                            const uint8_t *d_codes, const uint8_t *d_sf, float G_d, float *Y) {
  orc_nvfp4_gemv(h_codes, h_sf, Gh, d_codes, d_sf, G_d, H, F, Y);
}
