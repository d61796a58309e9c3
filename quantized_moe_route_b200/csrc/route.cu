// route.cu -- softmax + top-k routing, one warp per token.
//
// The router of "Drama 3 int4 (drama-rs format)" ("What's quantized": bf16
// router) scores 256 experts per token ("Drama 3 - NVFP4 routed experts",
// "Quantization"); the expert selection is softmax over all experts, top-k by
// logit (larger first, equal logits to the lower id first), and the selected
// probabilities renormalised to one.
#include "common.cuh"

namespace moe {

constexpr int kRouteMaxPerLane = 32;  // E <= 1024

// Lane l owns experts l, l + 32, l + 64, ... (coalesced loads).  Each of the
// k rounds takes the warp-wide maximum (value, then lowest id) of the
// not-yet-taken experts; only the winning lane rescans its own entries.
// Weights are exp(l_j - max) / sum over the selected of exp(l_j' - max): the
// renormalised softmax restricted to the selection.
template <int PER>
__global__ void route_kernel(const float *__restrict__ logits, int T, int E, int k,
                             int32_t *__restrict__ idx, float *__restrict__ w) {
  const int warps = blockDim.x / 32;
  const int t = blockIdx.x * warps + threadIdx.x / 32;
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  const float *l = logits + (size_t)t * E;
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? l[e] : -INFINITY;
  }
  uint32_t taken = 0;  // bit i: expert lane + 32 i already selected
  // local best of the untaken entries: entries visited in increasing id and
  // strict > keeps the lowest id among equals; -1 = nothing left
  auto local_best = [&](float &bv, int &bi) {
    bv = -INFINITY;
    bi = -1;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (bi < 0 || v[i] > bv)) {
        bv = v[i];
        bi = e;
      }
    }
  };
  float bv;
  int bi;
  local_best(bv, bi);
  float top = 0.f, denom = 0.f, my_w = 0.f;
  int my_idx = 0;
  for (int j = 0; j < k; ++j) {
    // warp arg-max: larger value, then lower id; exhausted lanes carry INT_MAX
    float rv = bv;
    int ri = bi < 0 ? 0x7fffffff : bi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, rv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, ri, o);
      if (oi != 0x7fffffff && (ri == 0x7fffffff || ov > rv || (ov == rv && oi < ri))) {
        rv = ov;
        ri = oi;
      }
    }
    if ((ri & 31) == lane) {
      taken |= 1u << (ri >> 5);
      local_best(bv, bi);
    }
    if (j == 0) top = rv;
    const float ex = expf(rv - top);
    denom += ex;
    if (lane == j) {
      my_idx = ri;
      my_w = ex;
    }
  }
  if (lane < k) {
    idx[(size_t)t * k + lane] = my_idx;
    w[(size_t)t * k + lane] = my_w / denom;
  }
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status moe_route(const float *logits, int T, int E, int k, int32_t *idx,
                                        float *w, moe_stream_t stream) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > 32 * kRouteMaxPerLane || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!logits || !idx || !w) return MOE_ERR_INVALID_ARG;
  const int threads = 128, warps = threads / 32;
  const dim3 grid((T + warps - 1) / warps);
  cudaStream_t s = as_stream(stream);
  const int per = (E + 31) / 32;
  if (per <= 1) route_kernel<1><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
  else if (per <= 2) route_kernel<2><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
  else if (per <= 4) route_kernel<4><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
  else if (per <= 8) route_kernel<8><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
  else if (per <= 16) route_kernel<16><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
  else route_kernel<32><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
  return launch_status();
}
