// combine.cu -- router-weighted combine of the k expert outputs of a token.
//
// y[t] = sum over j = 0..k-1 of w[t][j] * Y[p(t*k + j)], fp32 in that fixed j
// order, rounded to nearest-even bf16.  Each block owns whole output rows, so
// the "scatter" back to token order needs no atomics and is deterministic.
#include "common.cuh"

namespace moe {

// KC > 0 (bf16 rows only): k == KC is known at compile time, so the KC row
// indices, then the KC rows, are all requested before the in-order sum.
template <bool kBf16In, int KC = 0>
__global__ void combine_kernel(const void *__restrict__ Y, const int32_t *__restrict__ inv,
                               const float *__restrict__ w, int T, int k, int H,
                               uint16_t *__restrict__ y) {
  const int t = blockIdx.y;
  const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  grid_dep_wait();
  if (t >= T || c0 >= H) return;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  if (KC > 0) {
    size_t pr[KC > 0 ? KC : 1];
    float wr[KC > 0 ? KC : 1];
    uint4 q[KC > 0 ? KC : 1];
#pragma unroll
    for (int j = 0; j < KC; ++j) {
      const int r = t * KC + j;
      pr[j] = inv ? (size_t)inv[r] : (size_t)r;
      wr[j] = w[r];
    }
#pragma unroll
    for (int j = 0; j < KC; ++j) q[j] = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(Y) + pr[j] * H + c0);
#pragma unroll
    for (int j = 0; j < KC; ++j) {
      const uint32_t u[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(wr[j], __uint_as_float(u[i] << 16)));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(wr[j], __uint_as_float(u[i] & 0xFFFF0000u)));
      }
    }
  }
  for (int j = 0; KC == 0 && j < k; ++j) {
    const int r = t * k + j;
    const size_t p = inv ? (size_t)inv[r] : (size_t)r;
    const float wj = w[r];
    float v[8];
    if (kBf16In) {
      uint4 q = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(Y) + p * H + c0);
      const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(u[i] << 16);
        v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
    } else {
      const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(Y) + p * H + c0);
      float4 a = src[0], b = src[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(wj, v[i]));
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4 *>(y + (size_t)t * H + c0) = o;
  grid_dep_trigger();
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status moe_unpermute_combine(const void *Y, int y_dtype, const int32_t *inv,
                                                    const float *w, int T, int k, int H,
                                                    uint16_t *y, moe_stream_t stream) {
  if (T < 0 || k <= 0 || H <= 0 || (y_dtype != 0 && y_dtype != 1)) return MOE_ERR_INVALID_ARG;
  if (H % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!Y || !w || !y) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(Y) % 16 || reinterpret_cast<uintptr_t>(y) % 16)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T > 65535) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int threads = 128;
  dim3 grid((H / 8 + threads - 1) / threads, T);
  auto kern = y_dtype == 1 ? (k == 8 ? combine_kernel<true, 8> : combine_kernel<true>) : combine_kernel<false>;
  return launch_pdl(kern, grid, dim3(threads), 0, as_stream(stream), Y, inv, w, T, k, H, y);
}
