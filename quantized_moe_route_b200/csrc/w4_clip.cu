// w4_clip.cu -- int4 quantisers with the MSE clip search, and the symmetric
// group-128 int4 format packed for the same kernels.
//
// Sources: "Drama 3 int4 (drama-rs format)", table "What's quantized"
// (routed experts int4, asymmetric, group 64, f16 scale + min, MSE clip
// search); "drama-3-w4a16", section "How it was made" (round-to-nearest int4,
// one scale per 128 input weights, each scale chosen from 20 clipping ratios
// 1.0 -> 0.81 by minimum squared error) and table "At a glance" (int4,
// symmetric, group 128, GPTQ packing: zero point 8).
//
// Candidate i = 0..19 scales the group's range by p_i = (100 - i) / 100:
//   asymmetric g64: m = f16(p mn) toward -inf, s = f16((p mx - m) / 15) toward
//                   +inf, q = clamp(rint((w - m) / s), 0, 15), w^ = q s + m
//   symmetric g128: s = f16(2 (p amax) / 15) nearest-even,
//                   q = clamp(rint(w / s) + 8, 0, 15), w^ = (q - 8) s
// and the candidate with the smallest fp32 sum over the group, in channel
// order, of (w^ - w)^2 wins (ties to the smaller i).  Every operation is a
// single correctly rounded fp32 operation written out with _rn intrinsics,
// so the decision is the same on any device and in any build.
//
// A symmetric group-128 matrix runs through the int4 kernels unchanged: a
// group of 128 is two groups of 64 with scale s and min -8 s (exact in f16
// for s < 8192), and q s + (-8 s) = (q - 8) s exactly in fp32.
#include "common.cuh"

namespace moe {

constexpr int kClipRatios = 20;
constexpr int kClipGroupsPerBlock = 8;  // one warp per group

__device__ __forceinline__ float clip_ratio(int i) { return __fdiv_rn((float)(100 - i), 100.0f); }

// Lane c < 20 scores candidate c; the warp agrees on the best (smallest
// error, then smallest c) and writes the group with it.
template <bool kSym>
__global__ void __launch_bounds__(32 * kClipGroupsPerBlock)
    clip_search_kernel(const float *__restrict__ w, int N, int K, uint8_t *__restrict__ codes,
                       uint16_t *__restrict__ scale, uint16_t *__restrict__ minv) {
  constexpr int GS = kSym ? 128 : 64, PER = GS / 32;
  const int G = K / GS;
  const long long task = (long long)blockIdx.x * kClipGroupsPerBlock + threadIdx.x / 32;
  if (task >= (long long)N * G) return;
  const int lane = threadIdx.x & 31;
  const int n = (int)(task / G), g = (int)(task % G);
  const float *wg = w + (size_t)n * K + (size_t)g * GS;
  float v[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) v[j] = wg[lane + 32 * j];
  // the group's range
  float lo = v[0], hi = v[0];
#pragma unroll
  for (int j = 1; j < PER; ++j) {
    lo = fminf(lo, v[j]);
    hi = fmaxf(hi, v[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const float amax = fmaxf(fabsf(lo), fabsf(hi));

  // candidate of a ratio index: (scale, min) as f16 bits and fp32 values
  auto candidate = [&](int c, uint16_t *sb, uint16_t *mb, float *s, float *m) {
    const float p = clip_ratio(c);
    if (kSym) {
      const float t = __fmul_rn(2.0f, __fmul_rn(p, amax));
      const __half sh = __float2half_rn(__fdiv_rn(t, 15.0f));
      *sb = __half_as_ushort(sh);
      *s = __half2float(sh);
      *mb = 0;
      *m = 0.f;
    } else {
      const __half mh = __float2half_rd(__fmul_rn(p, lo));
      *m = __half2float(mh);
      const __half sh = __float2half_ru(__fdiv_rn(__fsub_rn(__fmul_rn(p, hi), *m), 15.0f));
      *s = __half2float(sh);
      *sb = __half_as_ushort(sh);
      *mb = __half_as_ushort(mh);
    }
  };
  auto code = [&](float x, float s, float m) {
    if (kSym) return s > 0.f ? fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(x, s)), 8.0f), 0.f), 15.f) : 8.f;
    return s > 0.f ? fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x, m), s)), 0.f), 15.f) : 0.f;
  };

  float err = __int_as_float(0x7f800000);  // +inf for the lanes without a candidate
  if (lane < kClipRatios) {
    uint16_t sb, mb;
    float s, m;
    candidate(lane, &sb, &mb, &s, &m);
    err = 0.f;
    for (int k = 0; k < GS; ++k) {  // channel order, as the sum is defined
      const float x = wg[k];
      const float q = code(x, s, m);
      const float deq = kSym ? __fmul_rn(__fsub_rn(q, 8.0f), s) : __fmaf_rn(q, s, m);
      const float d = __fsub_rn(deq, x);
      err = __fadd_rn(err, __fmul_rn(d, d));
    }
  }
  // smallest error, ties to the smallest ratio index
  float be = err;
  int bi = lane;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float oe = __shfl_xor_sync(0xffffffffu, be, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (oe < be || (oe == be && oi < bi)) {
      be = oe;
      bi = oi;
    }
  }
  uint16_t sb, mb;
  float s, m;
  candidate(bi, &sb, &mb, &s, &m);
  uint8_t *cg = codes + (size_t)n * K + (size_t)g * GS;
#pragma unroll
  for (int j = 0; j < PER; ++j) cg[lane + 32 * j] = (uint8_t)code(v[j], s, m);
  if (lane == 0) {
    scale[(size_t)n * G + g] = sb;
    if (!kSym) minv[(size_t)n * G + g] = mb;
  }
}

// Symmetric group-128 scales -> per-64-group (scale, min = -8 scale) pairs,
// then the ordinary packer.  One thread per (row, 64-group).
__global__ void sym128_affine_kernel(const uint16_t *__restrict__ scale128, int N, int K,
                                     uint16_t *__restrict__ scale64, uint16_t *__restrict__ min64) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int G = K / kGroup;
  if (t >= (long long)N * G) return;
  const int n = (int)(t / G), g = (int)(t % G);
  const uint16_t sb = scale128[(size_t)n * (K / 128) + g / 2];
  scale64[t] = sb;
  min64[t] = __half_as_ushort(__float2half_rn(__fmul_rn(-8.0f, f16_bits_to_f32(sb))));
}

template <bool kSym>
static moe_status clip_launch(const float *w, int N, int K, uint8_t *codes, uint16_t *scale,
                              uint16_t *minv, cudaStream_t stream) {
  const int GS = kSym ? 128 : 64;
  const long long tasks = (long long)N * (K / GS);
  const long long blocks = (tasks + kClipGroupsPerBlock - 1) / kClipGroupsPerBlock;
  clip_search_kernel<kSym><<<(unsigned)blocks, 32 * kClipGroupsPerBlock, 0, stream>>>(w, N, K, codes,
                                                                                      scale, minv);
  return launch_status();
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status moe_quantize_w4_clip(const float *w, int N, int K, uint8_t *codes,
                                                   uint16_t *scale, uint16_t *minv,
                                                   moe_stream_t stream) {
  if (N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (K % kGroup) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)N * K == 0) return MOE_OK;
  if (!w || !codes || !scale || !minv) return MOE_ERR_INVALID_ARG;
  return clip_launch<false>(w, N, K, codes, scale, minv, as_stream(stream));
}

extern "C" MOE_API moe_status moe_quantize_w4_sym128(const float *w, int N, int K, uint8_t *codes,
                                                     uint16_t *scale, moe_stream_t stream) {
  if (N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (K % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)N * K == 0) return MOE_OK;
  if (!w || !codes || !scale) return MOE_ERR_INVALID_ARG;
  return clip_launch<true>(w, N, K, codes, scale, nullptr, as_stream(stream));
}

extern "C" MOE_API size_t moe_pack_w4_sym128_workspace_bytes(int N, int K) {
  if (N <= 0 || K <= 0) return 0;
  return 2 * sizeof(uint16_t) * (size_t)N * (K / kGroup);
}

extern "C" MOE_API moe_status moe_pack_w4_sym128(const uint8_t *codes, const uint16_t *scale, int N,
                                                 int K, int kind, void *packed, size_t packed_bytes,
                                                 void *ws, size_t ws_bytes, moe_stream_t stream) {
  if (N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (K % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)N * K == 0) return MOE_OK;
  if (!codes || !scale) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_pack_w4_sym128_workspace_bytes(N, K)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 4) return MOE_ERR_INVALID_ARG;
  uint16_t *s64 = static_cast<uint16_t *>(ws);
  uint16_t *m64 = s64 + (size_t)N * (K / kGroup);
  const long long t = (long long)N * (K / kGroup);
  sym128_affine_kernel<<<(unsigned)((t + 255) / 256), 256, 0, as_stream(stream)>>>(scale, N, K, s64, m64);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  return moe_pack_w4(codes, s64, m64, N, K, kind, packed, packed_bytes, stream);
}
