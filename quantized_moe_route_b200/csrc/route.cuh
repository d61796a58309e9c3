// route.cuh -- warp-level softmax + top-k routing of one token, shared by
// the routing kernel and the fused decode kernel (identical results).
//
// The router of "Drama 3 int4 (drama-rs format)" ("What's quantized": bf16
// router) scores the routed experts ("Drama 3 - NVFP4 routed experts",
// "Quantization"); selection is top-k by logit (larger first, equal logits to
// the lower id first) and the weights are the selected softmax
// probabilities renormalised to one.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kRouteMaxPerLane = 32;  // E <= 1024

// One warp, one token.  Lane l owns experts l, l + 32, l + 64, ...
// (coalesced loads).  Each of the k rounds takes the warp-wide maximum
// (value, then lowest id) of the not-yet-taken experts; only the winning lane
// rescans its own entries.  Weights are exp(l_j - max) / sum over the
// selected of exp(l_j' - max): the renormalised softmax restricted to the
// selection.  Lane j < k returns the j-th selection in *idx_j, *w_j.
template <int PER>
__device__ __forceinline__ void route_token_warp(const float *__restrict__ l, int E, int k,
                                                 int *idx_j, float *w_j) {
  const int lane = threadIdx.x & 31;
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
  *idx_j = my_idx;
  *w_j = my_w / denom;
}

}  // namespace moe
