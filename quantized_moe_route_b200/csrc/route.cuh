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

// moe_route's kernel on finished logits (one warp per token), launched with
// programmatic dependent launch; for other launchers of the library
moe_status route_rows(const float *logits, int T, int E, int k, int32_t *idx, float *w, cudaStream_t stream);

// One warp, one token.  Lane l owns experts l, l + 32, l + 64, ...
// (coalesced loads).  Each of the k rounds takes the warp-wide maximum
// (value, then lowest id) of the not-yet-taken experts with two single-
// instruction warp reductions (max of an order-preserving integer key of the
// logit, then min of the ids holding that key); only the winning lane
// rescans its own entries.  Weights are exp(l_j - max) / sum over the
// selected of exp(l_j' - max): the renormalised softmax restricted to the
// selection.  Lane j < k returns the j-th selection in *idx_j, *w_j.

// Unsigned key ordered like the float (both zeros map to one key); 0 is
// below every finite logit and marks "nothing left".
__device__ __forceinline__ uint32_t route_key(float f) {
  const uint32_t b = f == 0.f ? 0u : __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float route_key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// The selection from the lanes' keys: key[i] is expert lane + 32 i's
// route_key (0 past the last expert).
//
// Eight entries per lane (E <= 256): each lane first sorts its entries by
// (key larger first, id smaller first) with a 19-comparator merge network,
// so a round's winner only shifts its list; the winner is the one lane whose
// head equals the warp maximum (a ballot), or, when several heads are equal,
// the lowest id among them (a second reduction).  The same selection as the
// general form, with a shorter dependent chain per round.  (A butterfly
// merge of the lanes' sorted lists, five exchange steps of eight 64-bit
// values, measured slower than these k rounds.)
template <int PER>
__device__ __forceinline__ void route_token_keys(const uint32_t (&key)[PER], int k, int *idx_j, float *w_j) {
  const int lane = threadIdx.x & 31;
  if constexpr (PER == 8) {
    uint64_t c[8];  // key << 8 | (255 - i): larger is earlier
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = ((uint64_t)key[i] << 8) | (uint64_t)(255 - i);
    auto cas = [&](int a, int b) {  // c[a] >= c[b] afterwards
      const uint64_t hi = c[a] > c[b] ? c[a] : c[b], lo = c[a] > c[b] ? c[b] : c[a];
      c[a] = hi;
      c[b] = lo;
    };
    cas(0, 1); cas(2, 3); cas(4, 5); cas(6, 7);
    cas(0, 2); cas(1, 3); cas(4, 6); cas(5, 7);
    cas(1, 2); cas(5, 6);
    cas(0, 4); cas(1, 5); cas(2, 6); cas(3, 7);
    cas(2, 4); cas(3, 5);
    cas(1, 2); cas(3, 4); cas(5, 6);
    float top = 0.f, denom = 0.f, my_w = 0.f;
    int my_idx = 0;
    for (int j = 0; j < k; ++j) {
      const uint32_t hk = (uint32_t)(c[0] >> 8);
      const uint32_t hid = (uint32_t)lane + 32u * (255u - (uint32_t)(c[0] & 0xFFu));
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, hk);
      const uint32_t hit = __ballot_sync(0xffffffffu, hk == kmax);
      uint32_t ri;
      int wl;
      if ((hit & (hit - 1u)) == 0u) {  // one lane holds the maximum
        wl = __ffs(hit) - 1;
        ri = __shfl_sync(0xffffffffu, hid, wl);
      } else {  // equal keys: the lowest id
        ri = __reduce_min_sync(0xffffffffu, hk == kmax ? hid : 0xffffffffu);
        wl = (int)(ri & 31u);
      }
      if (lane == wl) {
#pragma unroll
        for (int i = 0; i < 7; ++i) c[i] = c[i + 1];
        c[7] = 0ull;
      }
      const float rv = route_key_value(kmax);
      if (j == 0) top = rv;
      const float ex = expf(rv - top);
      denom += ex;
      if (lane == j) {
        my_idx = (int)ri;
        my_w = ex;
      }
    }
    *idx_j = my_idx;
    *w_j = my_w / denom;
    return;
  }
  uint32_t taken = 0;  // bit i: expert lane + 32 i already selected
  // local best of the untaken entries: entries visited in increasing id and
  // strict > keeps the lowest id among equal keys; key 0 = nothing left
  auto local_best = [&](uint32_t &bk, int &bi) {
    bk = 0u;
    bi = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (!((taken >> i) & 1u) && key[i] > bk) {
        bk = key[i];
        bi = lane + 32 * i;
      }
    }
  };
  uint32_t bk;
  int bi;
  local_best(bk, bi);
  float top = 0.f, denom = 0.f, my_w = 0.f;
  int my_idx = 0;
  for (int j = 0; j < k; ++j) {
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t ri = __reduce_min_sync(0xffffffffu, (bk == kmax && bk != 0u) ? (uint32_t)bi : 0xffffffffu);
    if ((int)(ri & 31u) == lane) {
      taken |= 1u << (ri >> 5);
      local_best(bk, bi);
    }
    const float rv = route_key_value(kmax);
    if (j == 0) top = rv;
    const float ex = expf(rv - top);
    denom += ex;
    if (lane == j) {
      my_idx = (int)ri;
      my_w = ex;
    }
  }
  *idx_j = my_idx;
  *w_j = my_w / denom;
}

template <int PER>
__device__ __forceinline__ void route_token_warp(const float *__restrict__ l, int E, int k,
                                                 int *idx_j, float *w_j) {
  const int lane = threadIdx.x & 31;
  uint32_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? route_key(l[e]) : 0u;
  }
  route_token_keys<PER>(key, k, idx_j, w_j);
}

}  // namespace moe
