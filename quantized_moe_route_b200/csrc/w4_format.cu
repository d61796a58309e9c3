// w4_format.cu -- int4 asymmetric group-64 expert weights: quantise, pack
// into the device layout, unpack, dequantise.
//
// Format: "Drama 3 int4 (drama-rs format)", section "What's quantized" (routed
// experts int4, asymmetric, group 64, f16 scale + min); weight = q*scale + min
// ("drama-rs", section "Apple Silicon (MLX)": packed affine form).
#include "common.cuh"

namespace moe {

// One warp per (row, group of 64): lane l holds channels l and l + 32.
__global__ void quantize_w4_kernel(const float *__restrict__ w, int N, int K,
                                   uint8_t *__restrict__ codes, uint16_t *__restrict__ scale,
                                   uint16_t *__restrict__ minv) {
  const int G = K / kGroup;
  const long long task = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (task >= (long long)N * G) return;
  const int lane = threadIdx.x & 31;
  const int n = (int)(task / G), g = (int)(task % G);
  const float *wg = w + (size_t)n * K + (size_t)g * kGroup;
  float a = wg[lane], b = wg[lane + 32];
  float mn = fminf(a, b), mx = fmaxf(a, b);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const __half mh = __float2half_rd(mn);
  const float m = __half2float(mh);
  const float span = __fsub_rn(mx, m);
  const __half sh = __float2half_ru(__fdiv_rn(span, 15.0f));
  const float s = __half2float(sh);
  float qa = 0.f, qb = 0.f;
  if (s > 0.f) {
    qa = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(a, m), s)), 0.f), 15.f);
    qb = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(b, m), s)), 0.f), 15.f);
  }
  uint8_t *cg = codes + (size_t)n * K + (size_t)g * kGroup;
  cg[lane] = (uint8_t)qa;
  cg[lane + 32] = (uint8_t)qb;
  if (lane == 0) {
    scale[(size_t)n * G + g] = __half_as_ushort(sh);
    minv[(size_t)n * G + g] = __half_as_ushort(mh);
  }
}

// One thread per (strip, group, lane): builds the 16 code bytes of that lane.
__global__ void pack_w4_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ scale,
                               const uint16_t *__restrict__ minv, int N, int K, int kind,
                               uint8_t *__restrict__ packed) {
  const int G = K / kGroup, S = N / kBlkRows;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= (long long)S * G * 32) return;
  const int lane = (int)(tid & 31);
  const long long blk = tid >> 5;
  const int s = (int)(blk / G), g = (int)(blk % G);
  const int row0 = w4_row_of_strip(s, N, kind);
  const int gi = lane >> 2, t = lane & 3;
  uint32_t words[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t wd = 0;
#pragma unroll
    for (int hi_row = 0; hi_row < 2; ++hi_row)
#pragma unroll
      for (int hi_k = 0; hi_k < 2; ++hi_k)
#pragma unroll
        for (int odd = 0; odd < 2; ++odd) {
          int r = gi + 8 * hi_row, c = 16 * j + 2 * t + odd + 8 * hi_k;
          uint32_t q = codes[(size_t)(row0 + r) * K + (size_t)g * kGroup + c] & 15u;
          wd |= q << (16 * odd + 8 * hi_k + 4 * hi_row);
        }
    words[j] = wd;
  }
  uint8_t *dst = packed + (size_t)blk * kBlkBytes;
  *reinterpret_cast<uint4 *>(dst + 16 * lane) = make_uint4(words[0], words[1], words[2], words[3]);
  if (lane < kBlkRows) {
    size_t si = (size_t)(row0 + lane) * G + g;
    uint32_t sm = (uint32_t)scale[si] | ((uint32_t)minv[si] << 16);
    *reinterpret_cast<uint32_t *>(dst + kBlkCodeBytes + 4 * lane) = sm;
  }
}

// One thread per canonical (row, channel): unpack and/or dequantise.
__global__ void unpack_w4_kernel(const uint8_t *__restrict__ packed, int N, int K, int kind,
                                 uint8_t *__restrict__ codes, uint16_t *__restrict__ scale,
                                 uint16_t *__restrict__ minv, float *__restrict__ deq) {
  const int G = K / kGroup;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= (long long)N * K) return;
  const int n = (int)(tid / K), k = (int)(tid % K);
  const int s = w4_strip_of_row(n - (n % kBlkRows), N, kind);
  const int r = n % kBlkRows, g = k / kGroup, c = k % kGroup;
  int lane, word, shift;
  w4_block_pos(r, c, &lane, &word, &shift);
  const uint8_t *blk = packed + ((size_t)s * G + g) * kBlkBytes;
  uint32_t wd = *reinterpret_cast<const uint32_t *>(blk + 16 * lane + 4 * word);
  uint32_t q = (wd >> shift) & 15u;
  uint32_t sm = *reinterpret_cast<const uint32_t *>(blk + kBlkCodeBytes + 4 * r);
  if (codes) codes[tid] = (uint8_t)q;
  if (c == 0) {
    if (scale) scale[(size_t)n * G + g] = (uint16_t)(sm & 0xFFFFu);
    if (minv) minv[(size_t)n * G + g] = (uint16_t)(sm >> 16);
  }
  if (deq) {
    float sf = f16_bits_to_f32((uint16_t)(sm & 0xFFFFu));
    float mf = f16_bits_to_f32((uint16_t)(sm >> 16));
    deq[tid] = __fmaf_rn((float)q, sf, mf);
  }
}

static moe_status check_shape(int N, int K, int kind) {
  if (N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (kind != MOE_W4_PLAIN && kind != MOE_W4_GATE_UP) return MOE_ERR_INVALID_ARG;
  if (N % kBlkRows || K % kGroup) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (kind == MOE_W4_GATE_UP && N % (2 * kBlkRows)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_w4_packed_bytes(int N, int K) {
  if (N <= 0 || K <= 0) return 0;
  return w4_packed_bytes(N, K);
}

extern "C" MOE_API moe_status moe_quantize_w4(const float *w, int N, int K, uint8_t *codes,
                                              uint16_t *scale, uint16_t *minv,
                                              moe_stream_t stream) {
  if (N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (K % kGroup) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)N * K == 0) return MOE_OK;
  if (!w || !codes || !scale || !minv) return MOE_ERR_INVALID_ARG;
  long long tasks = (long long)N * (K / kGroup);
  int threads = 256, per = threads / 32;
  long long blocks = (tasks + per - 1) / per;
  quantize_w4_kernel<<<(unsigned)blocks, threads, 0, as_stream(stream)>>>(w, N, K, codes, scale,
                                                                          minv);
  return launch_status();
}

extern "C" MOE_API moe_status moe_pack_w4(const uint8_t *codes, const uint16_t *scale,
                                          const uint16_t *minv, int N, int K, int kind,
                                          void *packed, size_t packed_bytes, moe_stream_t stream) {
  moe_status st = check_shape(N, K, kind);
  if (st != MOE_OK) return st;
  if ((long long)N * K == 0) return MOE_OK;
  if (!codes || !scale || !minv || !packed) return MOE_ERR_INVALID_ARG;
  if (packed_bytes < w4_packed_bytes(N, K)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(packed) % 16) return MOE_ERR_INVALID_ARG;
  long long threads_total = (long long)(N / kBlkRows) * (K / kGroup) * 32;
  int threads = 256;
  pack_w4_kernel<<<(unsigned)((threads_total + threads - 1) / threads), threads, 0,
                   as_stream(stream)>>>(codes, scale, minv, N, K, kind,
                                        static_cast<uint8_t *>(packed));
  return launch_status();
}

static moe_status unpack_common(const void *packed, int N, int K, int kind, uint8_t *codes,
                                uint16_t *scale, uint16_t *minv, float *deq, moe_stream_t stream) {
  moe_status st = check_shape(N, K, kind);
  if (st != MOE_OK) return st;
  if ((long long)N * K == 0) return MOE_OK;
  if (!packed) return MOE_ERR_INVALID_ARG;
  long long total = (long long)N * K;
  int threads = 256;
  unpack_w4_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, as_stream(stream)>>>(
      static_cast<const uint8_t *>(packed), N, K, kind, codes, scale, minv, deq);
  return launch_status();
}

extern "C" MOE_API moe_status moe_unpack_w4(const void *packed, int N, int K, int kind,
                                            uint8_t *codes, uint16_t *scale, uint16_t *minv,
                                            moe_stream_t stream) {
  if (!codes || !scale || !minv) return MOE_ERR_INVALID_ARG;
  return unpack_common(packed, N, K, kind, codes, scale, minv, nullptr, stream);
}

extern "C" MOE_API moe_status moe_dequant_w4(const void *packed, int N, int K, int kind, float *out,
                                             moe_stream_t stream) {
  if (!out) return MOE_ERR_INVALID_ARG;
  return unpack_common(packed, N, K, kind, nullptr, nullptr, nullptr, out, stream);
}
