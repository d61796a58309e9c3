// route.cu -- softmax + top-k routing, one warp per token.
//
// The router of "Drama 3 int4 (drama-rs format)" ("What's quantized": bf16
// router) scores 256 experts per token ("Drama 3 - NVFP4 routed experts",
// "Quantization"); the expert selection is softmax over all experts, top-k by
// logit (larger first, equal logits to the lower id first), and the selected
// probabilities renormalised to one.
#include "route.cuh"

namespace moe {

// shared != 0: each token's row has k + 1 entries, the last one the shared
// expert (id E) with weight 1
template <int PER>
__global__ void route_kernel(const float *__restrict__ logits, int T, int E, int k, int shared,
                             int32_t *__restrict__ idx, float *__restrict__ w) {
  const int warps = blockDim.x / 32;
  const int t = blockIdx.x * warps + threadIdx.x / 32;
  grid_dep_wait();
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  int my_idx;
  float my_w;
  route_token_warp<PER>(logits + (size_t)t * E, E, k, &my_idx, &my_w);
  const int kk = k + shared;
  if (lane < k) {
    idx[(size_t)t * kk + lane] = my_idx;
    w[(size_t)t * kk + lane] = my_w;
  } else if (shared && lane == k) {
    idx[(size_t)t * kk + k] = E;
    w[(size_t)t * kk + k] = 1.0f;
  }
  grid_dep_trigger();
}

static moe_status route_launch(const float *logits, int T, int E, int k, int shared, int32_t *idx,
                               float *w, moe_stream_t stream) {
  const int threads = 128, warps = threads / 32;
  const dim3 grid((T + warps - 1) / warps);
  cudaStream_t s = as_stream(stream);
  const int per = (E + 31) / 32;
  auto kern = per <= 1 ? route_kernel<1> : per <= 2 ? route_kernel<2> : per <= 4 ? route_kernel<4>
             : per <= 8 ? route_kernel<8> : per <= 16 ? route_kernel<16> : route_kernel<32>;
  return launch_pdl(kern, grid, dim3(threads), 0, s, logits, T, E, k, shared, idx, w);
}

moe_status route_rows(const float *logits, int T, int E, int k, int32_t *idx, float *w, cudaStream_t stream) {
  return route_launch(logits, T, E, k, 0, idx, w, reinterpret_cast<moe_stream_t>(stream));
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status moe_route(const float *logits, int T, int E, int k, int32_t *idx,
                                        float *w, moe_stream_t stream) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > 32 * kRouteMaxPerLane || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!logits || !idx || !w) return MOE_ERR_INVALID_ARG;
  return route_launch(logits, T, E, k, 0, idx, w, stream);
}

extern "C" MOE_API moe_status moe_route_shared(const float *logits, int T, int E, int k, int32_t *idx,
                                               float *w, moe_stream_t stream) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > 32 * kRouteMaxPerLane - 1 || k > 31) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!logits || !idx || !w) return MOE_ERR_INVALID_ARG;
  return route_launch(logits, T, E, k, 1, idx, w, stream);
}
