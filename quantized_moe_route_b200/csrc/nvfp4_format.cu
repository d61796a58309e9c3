// nvfp4_format.cu -- NVFP4 expert weights and activations: global scale,
// quantise, pack into the device layout, unpack; per-row activation
// quantisation.
//
// Format: "Drama 3 - NVFP4 routed experts", section "Quantization": E2M1
// codes, one E4M3 scale per 16 input channels, one FP32 global scale per
// matrix (gate and up share theirs), round to nearest; activations get a
// dynamic per-token FP32 global with E4M3 block scales.
//   G      = amax / (448 * 6)          (1 when amax == 0)
//   S_b    = E4M3(amax_b / (6 G))      nearest-even, saturating at 448
//   code_i = E2M1(v_i / (S_b G))       nearest-even, saturating at 6 (0 if S_b == 0)
// Every division and product is one correctly rounded fp32 operation, in the
// order written, so a code depends only on its fp32 inputs.  The E4M3 and
// E2M1 conversions are CUDA's own (cuda_fp8.h / cuda_fp4.h).
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "nvfp4.cuh"

namespace moe {

__device__ __forceinline__ uint8_t e4m3_rne_sat(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ uint8_t e2m1_rne_sat(float v) {
  return (uint8_t)__nv_cvt_float_to_fp4(v, __NV_E2M1, cudaRoundNearest) & 15u;
}

// One 16-value block: its E4M3 scale and 16 codes (one per byte).
__device__ __forceinline__ uint8_t nvfp4_block(const float (&v)[16], float G, uint8_t (&c)[16]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint8_t s8 = e4m3_rne_sat(__fdiv_rn(amax, __fmul_rn(6.0f, G)));
  const float sb = e4m3_to_f32(s8);
  const float scale = __fmul_rn(sb, G);
#pragma unroll
  for (int i = 0; i < 16; ++i) c[i] = sb == 0.f ? (uint8_t)0 : e2m1_rne_sat(__fdiv_rn(v[i], scale));
  return s8;
}

// G <- max |v| over n values, as the bit pattern of a non-negative float
// (ordered like unsigned integers); G must hold 0 on entry.
__global__ void amax_kernel(const float *__restrict__ v, size_t n, float *G) {
  float m = 0.f;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned int *>(G), __float_as_uint(m));
}
__global__ void global_finish_kernel(float *G) {
  const float amax = *G;
  *G = amax == 0.f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// One thread per (row, 16-block) of a matrix with a given global.
__global__ void quantize_nvfp4_kernel(const float *__restrict__ v, int N, int K,
                                      const float *__restrict__ Gp, uint8_t *__restrict__ codes,
                                      uint8_t *__restrict__ sf) {
  const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nb = K / 16;
  if (b >= (long long)N * nb) return;
  const float G = *Gp;
  const float4 *src = reinterpret_cast<const float4 *>(v + b * 16);
  float x[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 q = src[i];
    x[4 * i] = q.x, x[4 * i + 1] = q.y, x[4 * i + 2] = q.z, x[4 * i + 3] = q.w;
  }
  uint8_t c[16];
  sf[b] = nvfp4_block(x, G, c);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = c[4 * i] | (c[4 * i + 1] << 8) | (c[4 * i + 2] << 16) | ((uint32_t)c[4 * i + 3] << 24);
  *reinterpret_cast<uint4 *>(codes + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
}

// One thread per packed byte of a strip (codes, then scales).
__global__ void pack_nvfp4_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ sf,
                                  int N, int K, int kind, uint8_t *__restrict__ packed) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long strip_bytes = nvfp4_strip_bytes(K);
  if (i >= (long long)(N / kBlkRows) * strip_bytes) return;
  const int s = (int)(i / strip_bytes);
  const int o = (int)(i % strip_bytes);
  const int row0 = w4_row_of_strip(s, N, kind);
  if (o < kBlkRows * K / 2) {
    // invert nvfp4_code_pos: the XOR permutation is its own inverse
    const int r = o / (K / 2), p = o % (K / 2);
    const int b = (p & ~127) + ((((p >> 4) & 7) ^ (r & 7)) << 4) + (p & 15);
    const uint8_t *c = codes + (size_t)(row0 + r) * K + 2 * b;
    packed[i] = (uint8_t)((c[0] & 15u) | ((c[1] & 15u) << 4));
  } else {
    const int q = o - kBlkRows * K / 2;  // = (blk >> 2) * 64 + r * 4 + (blk & 3)
    const int r = (q % 64) / 4, blk = (q / 64) * 4 + (q % 4);
    packed[i] = sf[(size_t)(row0 + r) * (K / 16) + blk];
  }
}

// One thread per canonical (row, 16-block).
__global__ void unpack_nvfp4_kernel(const uint8_t *__restrict__ packed, int N, int K, int kind,
                                    uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
  const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nb = K / 16;
  if (b >= (long long)N * nb) return;
  const int n = (int)(b / nb), blk = (int)(b % nb);
  const int s = w4_strip_of_row(n - n % kBlkRows, N, kind), r = n % kBlkRows;
  const uint8_t *strip = packed + (size_t)s * nvfp4_strip_bytes(K);
  for (int i = 0; i < 8; ++i) {
    const uint8_t v = strip[nvfp4_code_pos(r, 8 * blk + i, K)];
    codes[b * 16 + 2 * i] = v & 15u;
    codes[b * 16 + 2 * i + 1] = v >> 4;
  }
  sf[b] = strip[kBlkRows * (K / 2) + nvfp4_scale_pos(r, blk)];
}

// One warp per output row p: source row src = rows ? rows[p] / div : p.
// Pass 1: row amax -> G; pass 2 (lane per 16-block): scale and codes,
// packed two per byte (channel 2i in the low nibble).
template <bool kF32>
__global__ void quantize_rows_kernel(const void *__restrict__ xv, int R, int K,
                                     const int32_t *__restrict__ rows, int div,
                                     uint8_t *__restrict__ codes, uint8_t *__restrict__ sf,
                                     float *__restrict__ Gout) {
  const int p = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  grid_dep_wait();
  if (p >= R) return;
  const int src = rows ? rows[p] / div : p;
  const int nb = K / 16;
  auto load16 = [&](int blk, float (&v)[16]) {
    if (kF32) {
      const float4 *q = reinterpret_cast<const float4 *>(static_cast<const float *>(xv) +
                                                         (size_t)src * K + 16 * blk);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 a = q[i];
        v[4 * i] = a.x, v[4 * i + 1] = a.y, v[4 * i + 2] = a.z, v[4 * i + 3] = a.w;
      }
    } else {
      const uint4 *q = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(xv) +
                                                       (size_t)src * K + 16 * blk);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 a = q[i];
        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * i + 2 * j] = __uint_as_float(u[j] << 16);
          v[8 * i + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
      }
    }
  };
  float amax = 0.f;
  for (int blk = lane; blk < nb; blk += 32) {
    float v[16];
    load16(blk, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float G = amax == 0.f ? 1.0f : __fdiv_rn(amax, 2688.0f);
  if (lane == 0) Gout[p] = G;
  for (int blk = lane; blk < nb; blk += 32) {
    float v[16];
    load16(blk, v);
    uint8_t c[16];
    sf[(size_t)p * nb + blk] = nvfp4_block(v, G, c);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i / 4] |= (uint32_t)(c[2 * i] | (c[2 * i + 1] << 4)) << (8 * (i % 4));
    *reinterpret_cast<uint2 *>(codes + (size_t)p * (K / 2) + 8 * blk) = make_uint2(w[0], w[1]);
  }
  grid_dep_trigger();
}

static moe_status nvfp4_check_shape(int N, int K, int kind) {
  if (N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (kind != MOE_W4_PLAIN && kind != MOE_W4_GATE_UP) return MOE_ERR_INVALID_ARG;
  if (N % kBlkRows || K % 256) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (kind == MOE_W4_GATE_UP && N % (2 * kBlkRows)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_nvfp4_packed_bytes(int N, int K) {
  if (N <= 0 || K <= 0) return 0;
  return (size_t)(N / kBlkRows) * nvfp4_strip_bytes(K);
}

extern "C" MOE_API moe_status moe_nvfp4_global(const float *v, size_t n, float *G,
                                               moe_stream_t stream) {
  if (!G || (n && !v)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaMemsetAsync(G, 0, sizeof(float), s);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  if (n) {
    const size_t blocks = (n + 255) / 256;
    amax_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(v, n, G);
    moe_status st = launch_status();
    if (st != MOE_OK) return st;
  }
  global_finish_kernel<<<1, 1, 0, s>>>(G);
  return launch_status();
}

extern "C" MOE_API moe_status moe_quantize_nvfp4(const float *v, int N, int K, const float *G,
                                                 uint8_t *codes, uint8_t *sf,
                                                 moe_stream_t stream) {
  if (N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (K % 16) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)N * K == 0) return MOE_OK;
  if (!v || !G || !codes || !sf) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(v) % 16 || reinterpret_cast<uintptr_t>(codes) % 16)
    return MOE_ERR_INVALID_ARG;
  const long long blocks = (long long)N * (K / 16);
  quantize_nvfp4_kernel<<<(unsigned)((blocks + 255) / 256), 256, 0, as_stream(stream)>>>(
      v, N, K, G, codes, sf);
  return launch_status();
}

extern "C" MOE_API moe_status moe_pack_nvfp4(const uint8_t *codes, const uint8_t *sf, int N, int K,
                                             int kind, void *packed, size_t packed_bytes,
                                             moe_stream_t stream) {
  moe_status st = nvfp4_check_shape(N, K, kind);
  if (st != MOE_OK) return st;
  if ((long long)N * K == 0) return MOE_OK;
  if (!codes || !sf || !packed) return MOE_ERR_INVALID_ARG;
  if (packed_bytes < moe_nvfp4_packed_bytes(N, K)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(packed) % 16) return MOE_ERR_INVALID_ARG;
  const long long total = (long long)moe_nvfp4_packed_bytes(N, K);
  pack_nvfp4_kernel<<<(unsigned)((total + 255) / 256), 256, 0, as_stream(stream)>>>(
      codes, sf, N, K, kind, static_cast<uint8_t *>(packed));
  return launch_status();
}

extern "C" MOE_API moe_status moe_unpack_nvfp4(const void *packed, int N, int K, int kind,
                                               uint8_t *codes, uint8_t *sf, moe_stream_t stream) {
  moe_status st = nvfp4_check_shape(N, K, kind);
  if (st != MOE_OK) return st;
  if ((long long)N * K == 0) return MOE_OK;
  if (!packed || !codes || !sf) return MOE_ERR_INVALID_ARG;
  const long long blocks = (long long)N * (K / 16);
  unpack_nvfp4_kernel<<<(unsigned)((blocks + 255) / 256), 256, 0, as_stream(stream)>>>(
      static_cast<const uint8_t *>(packed), N, K, kind, codes, sf);
  return launch_status();
}

extern "C" MOE_API moe_status moe_quantize_nvfp4_rows(const void *x, int x_dtype, int rows, int K,
                                                      const int32_t *src_rows, int src_div,
                                                      uint8_t *codes, uint8_t *sf, float *G,
                                                      moe_stream_t stream) {
  if (rows < 0 || K < 0 || (x_dtype != 0 && x_dtype != 1)) return MOE_ERR_INVALID_ARG;
  if (src_rows && src_div <= 0) return MOE_ERR_INVALID_ARG;
  if (K % 16) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)rows * K == 0) return MOE_OK;
  if (!x || !codes || !sf || !G) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(codes) % 8)
    return MOE_ERR_INVALID_ARG;
  const int warps = 8;
  const unsigned grid = (unsigned)((rows + warps - 1) / warps);
  return launch_pdl(x_dtype == 0 ? quantize_rows_kernel<false> : quantize_rows_kernel<true>, dim3(grid),
                    dim3(32 * warps), 0, as_stream(stream), x, rows, K, src_rows, src_div, codes, sf, G);
}
