// synth_gen.cu -- CUDA twin of synth/__init__.py's seeded input generator.
//
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11), one call per element;
// the four outputs cut to 24 bits are summed, centred, converted to fp32 with
// round-to-nearest-even and multiplied by one fp32 constant supplied by the
// host.  No part of the MoE method is computed here: this only draws inputs.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ void philox_round(uint32_t c[4], uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  uint32_t hi0 = __umulhi(M0, c[0]), lo0 = M0 * c[0];
  uint32_t hi1 = __umulhi(M1, c[2]), lo1 = M1 * c[2];
  uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
  c[0] = n0;
  c[1] = lo1;
  c[2] = n2;
  c[3] = lo0;
}

__device__ __forceinline__ float draw(uint64_t i, uint32_t a, uint32_t b, uint32_t seed,
                                      float scale) {
  uint32_t c[4] = {(uint32_t)i, (uint32_t)(i >> 32), a, b};
  uint32_t k0 = seed, k1 = 0x5EEDC0DEu;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    philox_round(c, k0, k1);
  }
  int s = (int)(c[0] >> 8) + (int)(c[1] >> 8) + (int)(c[2] >> 8) + (int)(c[3] >> 8) - (1 << 25);
  return __fmul_rn(__int2float_rn(s), scale);
}

// out[m][i] for m in [0, count), i in [0, n): stream a = a0 + a_step * m, b.
__global__ void normal_kernel(float *out, uint64_t n, int count, uint32_t a0, uint32_t a_step,
                              uint32_t b, uint32_t seed, float scale, uint64_t start) {
  const uint64_t total = n * (uint64_t)count;
  for (uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t m = t / n, i = t % n;
    out[t] = draw(start + i, a0 + a_step * (uint32_t)m, b, seed, scale);
  }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int synth_normal_f32(
    float *out, uint64_t n, int count, uint32_t a0, uint32_t a_step, uint32_t b, uint32_t seed,
    float scale, uint64_t start, void *stream) {
  if (n == 0 || count <= 0) return 0;
  normal_kernel<<<148 * 8, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      out, n, count, a0, a_step, b, seed, scale, start);
  return (int)cudaGetLastError();
}
