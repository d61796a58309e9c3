// router.cu -- the router linear fused with routing: logits = Wr x (bf16
// operands, fp32 sums, no bias) for every token, then softmax top-k with
// renormalised weights, in one launch.
//
// Source: the router stays bf16 ("Drama 3 int4 (drama-rs format)", table
// "What's quantized"; "DRAMA-3 MLX expert-only 4-bit", section "Quantization
// and provenance"); the routing is moe_route's (route.cuh).
//
// A CTA computes a tile of 16 tokens x TN experts (TN = 64 with four warps,
// or 16 with one warp for decode-sized batches, so that more CTAs share the
// router weights) on the tensor cores: m16n8k16 bf16 MMAs, fp32 accumulation,
// K in chunks of 64 channels staged through shared memory by cp.async (two
// stages).  It writes its logits, then counts one arrival for its token tile;
// the CTA whose arrival completes the tile's count routes those 16 tokens
// from the finished logits (read from L2) and resets the count to zero for
// the next call.  No CTA waits on another.
#include "common.cuh"
#include "route.cuh"

namespace moe {

constexpr int kRtTok = 16;   // tokens per tile (MMA M)
constexpr int kRtKc = 64;    // channels per K chunk
constexpr int kRtLd = kRtKc + 8;  // padded row (bf16): 144 bytes, conflict-free fragment loads

struct RouterArgs {
  const uint16_t *x;   // bf16 [T][H]
  const uint16_t *wr;  // bf16 [E][H]
  float *logits;       // [T][E]
  int32_t *idx;        // [T][k]
  float *w;            // [T][k]
  int *cnt;            // [ceil(T / 16)] arrival counts, zero between calls
  int T, E, H, k, tn;  // tn: experts per tile
};

__device__ __forceinline__ void cp_async_16z(void *dst, const void *src, bool valid) {
  // zero-fills the 16 bytes when !valid (no bytes are read then)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ int atom_add_acq_rel_gpu_rt(int *p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

template <int NW, int PER>
__global__ void __launch_bounds__(NW * 32) router_kernel(RouterArgs a) {
  constexpr int TN = 16 * NW;
  __shared__ __align__(16) uint16_t xs[2][kRtTok][kRtLd];
  __shared__ __align__(16) uint16_t ws[2][TN][kRtLd];
  __shared__ __align__(16) float lrow[NW][kRouteMaxPerLane * 32];  // one token's logits per warp
  __shared__ int last_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gi = lane >> 2, t4 = lane & 3;
  const int t0 = blockIdx.x * kRtTok, e0 = blockIdx.y * TN;
  const int T = a.T, E = a.E, H = a.H;
  const int nk = H / kRtKc;

  asm volatile("griddepcontrol.wait;" ::: "memory");
  auto load = [&](int kc, int s) {
    // x: 16 rows x 8 pieces of 16 bytes; Wr: TN rows x 8 pieces
    for (int v = tid; v < kRtTok * 8; v += NW * 32) {
      const int r = v >> 3, p = v & 7;
      const bool ok = t0 + r < T;
      cp_async_16z(&xs[s][r][8 * p], a.x + (size_t)(ok ? t0 + r : 0) * H + kc * kRtKc + 8 * p, ok);
    }
    for (int v = tid; v < TN * 8; v += NW * 32) {
      const int r = v >> 3, p = v & 7;
      cp_async_16z(&ws[s][r][8 * p], a.wr + (size_t)(e0 + r) * H + kc * kRtKc + 8 * p, true);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float acc[2][4] = {};
  load(0, 0);
  for (int kc = 0; kc < nk; ++kc) {
    const int s = kc & 1;
    if (kc + 1 < nk) {
      load(kc + 1, s ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kRtKc; kk += 16) {
      uint32_t af[4];
      af[0] = *reinterpret_cast<const uint32_t *>(&xs[s][gi][kk + 2 * t4]);
      af[1] = *reinterpret_cast<const uint32_t *>(&xs[s][gi + 8][kk + 2 * t4]);
      af[2] = *reinterpret_cast<const uint32_t *>(&xs[s][gi][kk + 2 * t4 + 8]);
      af[3] = *reinterpret_cast<const uint32_t *>(&xs[s][gi + 8][kk + 2 * t4 + 8]);
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const int n = 16 * warp + 8 * nb + gi;  // this lane's B column (expert in the tile)
        const uint32_t b0 = *reinterpret_cast<const uint32_t *>(&ws[s][n][kk + 2 * t4]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t *>(&ws[s][n][kk + 2 * t4 + 8]);
        mma_bf16_16816(acc[nb], af, b0, b1);
      }
    }
    __syncthreads();  // this stage is free for the chunk after next
  }

  // logits of the tile: rows gi, gi + 8 (tokens), columns 2 t4, 2 t4 + 1 of each n8 block
#pragma unroll
  for (int nb = 0; nb < 2; ++nb) {
    const int e = e0 + 16 * warp + 8 * nb + 2 * t4;
    if (t0 + gi < T) *reinterpret_cast<float2 *>(a.logits + (size_t)(t0 + gi) * E + e) = make_float2(acc[nb][0], acc[nb][1]);
    if (t0 + gi + 8 < T)
      *reinterpret_cast<float2 *>(a.logits + (size_t)(t0 + gi + 8) * E + e) = make_float2(acc[nb][2], acc[nb][3]);
  }
  // count this tile's arrival (the barrier orders the CTA's stores before the
  // releasing add); the arrival that completes the count routes the tokens
  __syncthreads();
  if (tid == 0) {
    const int old = atom_add_acq_rel_gpu_rt(&a.cnt[blockIdx.x], 1);
    last_s = old == (int)gridDim.y - 1;
    if (last_s) a.cnt[blockIdx.x] = 0;  // ready for the next call
  }
  __syncthreads();
  if (last_s) {
    for (int t = t0 + warp; t < min(T, t0 + kRtTok); t += NW) {
      for (int e = lane; e < E; e += 32) lrow[warp][e] = __ldcg(a.logits + (size_t)t * E + e);
      __syncwarp();
      int j_idx;
      float j_w;
      route_token_warp<PER>(lrow[warp], E, a.k, &j_idx, &j_w);
      if (lane < a.k) {
        a.idx[(size_t)t * a.k + lane] = j_idx;
        a.w[(size_t)t * a.k + lane] = j_w;
      }
      __syncwarp();
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int NW, int PER>
static moe_status router_launch(const RouterArgs &a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.T + kRtTok - 1) / kRtTok, a.E / (16 * NW));
  cfg.blockDim = dim3(32 * NW);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, router_kernel<NW, PER>, a);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

static size_t router_cnt_bytes(int T) { return ((size_t)((T + kRtTok - 1) / kRtTok) * 4 + 255) / 256 * 256; }

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_router_route_workspace_bytes(int T, int E) {
  if (T <= 0 || E <= 0) return 0;
  return router_cnt_bytes(T) + sizeof(float) * (size_t)T * E;
}

extern "C" MOE_API moe_status moe_router_route(const uint16_t *x, const uint16_t *wr, int T, int E, int H, int k,
                                               float *logits, int32_t *idx, float *w, void *ws, size_t ws_bytes,
                                               moe_stream_t stream) {
  if (T < 0 || E <= 0 || H <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (E % 16 || (E > 64 && E % 64) || H % kRtKc || E > 32 * kRouteMaxPerLane || k > 32)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x || !wr || !idx || !w) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(wr) % 16 ||
      reinterpret_cast<uintptr_t>(ws) % 16 || reinterpret_cast<uintptr_t>(logits) % 8)
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_router_route_workspace_bytes(T, E)) return MOE_ERR_WORKSPACE;
  RouterArgs a;
  a.x = x;
  a.wr = wr;
  a.cnt = static_cast<int *>(ws);
  a.logits = logits ? logits : reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + router_cnt_bytes(T));
  a.idx = idx;
  a.w = w;
  a.T = T;
  a.E = E;
  a.H = H;
  a.k = k;
  cudaStream_t s = as_stream(stream);
  // decode-sized batches: tiles of 16 experts (one warp), so the router
  // weights are shared by E / 16 CTAs; otherwise 64 experts (four warps)
  const bool narrow = T <= 64 || E < 64;
  a.tn = narrow ? 16 : 64;
  if (E <= 256) return narrow ? router_launch<1, 8>(a, s) : router_launch<4, 8>(a, s);
  return narrow ? router_launch<1, 32>(a, s) : router_launch<4, 32>(a, s);
}
