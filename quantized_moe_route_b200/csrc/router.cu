// router.cu -- the router linear fused with routing: logits = Wr x (bf16
// operands, fp32 sums, no bias) for every token, then softmax top-k with
// renormalised weights.
//
// Source: the router stays bf16 ("Drama 3 int4 (drama-rs format)", table
// "What's quantized"; "DRAMA-3 MLX expert-only 4-bit", section "Quantization
// and provenance"); the routing is moe_route's (route.cuh).
//
// Up to 16 tokens (decode), one launch: the router matrix is read once,
// spread over ceil(E / 2) CTAs.  A CTA holds two experts' rows; each lane
// takes 8 consecutive channels per 2048 (one 16-byte load per row) and sums
// the products of every token in fp32 FMAs; the lanes' sums meet in a
// shuffle tree and the warps' in shared memory in warp order, so the logits
// do not depend on scheduling.  One arrival count over the grid: its last CTA
// routes the tokens, one warp per token.
//
// More tokens: a tensor-core GEMM writes the logits, then the routing kernel
// of moe_route runs one warp per token (a second launch, chained by
// programmatic dependent launch).  A CTA of four warps computes a tile of BM
// tokens x 64 experts (BM = 64 from 256 tokens up, so every router row is
// read T / 64 times; 16 below, for more CTAs): m16n8k16 bf16 MMAs with
// ldmatrix fragments, fp32 accumulation, K in chunks of 64 channels staged
// through shared memory by cp.async with 8 (64-token tiles) or 6 chunks in
// flight.  Routing
// in the GEMM's last CTA per tile would serialise BM tokens on four warps;
// the separate launch routes every token in parallel.
#include <atomic>

#include "common.cuh"
#include "route.cuh"

namespace moe {

constexpr int kRtTok = 16;   // tokens per arrival counter (workspace sizing)
constexpr int kRtKc = 64;    // channels per K chunk
constexpr int kRtLd = kRtKc + 8;  // padded row (bf16): 144 bytes, conflict-free fragment loads
constexpr int kGvRows = 2;    // experts per CTA of the small-batch form
constexpr int kGvWarps = 16;  // one routing warp per token
constexpr int kGvMaxTok = 16;

struct RouterArgs {
  const uint16_t *x;   // bf16 [T][H]
  const uint16_t *wr;  // bf16 [E][H]
  float *logits;       // [T][E]
  int32_t *idx;        // [T][k]
  float *w;            // [T][k]
  int *cnt;            // arrival count of the small-batch form, zero between calls
  int T, E, H, k;
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

// the last arriver of a group of CTAs: true in every thread of the CTA whose
// arrival completes the count (the count is reset for the next call); the
// barrier before the releasing add orders the CTA's logit stores before it
__device__ __forceinline__ bool last_arrival(int *cnt, int expected, int *flag_s) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atom_add_acq_rel_gpu_rt(cnt, 1);
    *flag_s = old == expected - 1;
    if (*flag_s) *cnt = 0;  // ready for the next call
  }
  __syncthreads();
  return *flag_s != 0;
}

// warp-per-token routing of tokens t0 .. t1 - 1 from finished logits
template <int PER>
__device__ __forceinline__ void route_tokens(const RouterArgs &a, int t0, int t1, float *lrow, int nwarps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *row = lrow + warp * (PER * 32);
  for (int t = t0 + warp; t < t1; t += nwarps) {
    for (int e = lane; e < a.E; e += 32) row[e] = __ldcg(a.logits + (size_t)t * a.E + e);
    __syncwarp();
    int j_idx;
    float j_w;
    route_token_warp<PER>(row, a.E, a.k, &j_idx, &j_w);
    if (lane < a.k) {
      a.idx[(size_t)t * a.k + lane] = j_idx;
      a.w[(size_t)t * a.k + lane] = j_w;
    }
    __syncwarp();
  }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float f[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// small batches (T <= 16): two experts per CTA, CUDA-core FMAs
template <int PER>
__global__ void __launch_bounds__(kGvWarps * 32) router_gemv_kernel(RouterArgs a) {
  __shared__ float part[kGvWarps][kGvRows][kGvMaxTok];
  extern __shared__ __align__(16) float lrow[];  // [kGvWarps][PER * 32]: one token's logits per warp
  __shared__ int last_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, E = a.E, H = a.H;
  const int e0 = blockIdx.x * kGvRows;
  float acc[kGvRows][kGvMaxTok];
#pragma unroll
  for (int r = 0; r < kGvRows; ++r)
#pragma unroll
    for (int t = 0; t < kGvMaxTok; ++t) acc[r][t] = 0.f;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int c = 8 * tid; c < H; c += 8 * kGvWarps * 32) {
    float wf[kGvRows][8];
#pragma unroll
    for (int r = 0; r < kGvRows; ++r) {
      const int e = min(e0 + r, E - 1);  // a missing last row repeats a real one (never stored)
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(a.wr + (size_t)e * H + c)), wf[r]);
    }
    // every token's 16 bytes requested before the first product
    uint4 xv[kGvMaxTok];
#pragma unroll
    for (int t = 0; t < kGvMaxTok; ++t)
      if (t < T) xv[t] = __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)t * H + c));
#pragma unroll
    for (int t = 0; t < kGvMaxTok; ++t) {
      if (t < T) {
        float xf[8];
        bf16x8_to_f32(xv[t], xf);
#pragma unroll
        for (int r = 0; r < kGvRows; ++r)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[r][t] = __fmaf_rn(xf[i], wf[r][i], acc[r][t]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kGvRows; ++r)
#pragma unroll
    for (int t = 0; t < kGvMaxTok; ++t) {
      if (t < T) {
        float v = acc[r][t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) part[warp][r][t] = v;
      }
    }
  __syncthreads();
  if (tid < kGvRows * T) {
    const int r = tid / T, t = tid % T;
    float v = part[0][r][t];
#pragma unroll
    for (int w = 1; w < kGvWarps; ++w) v = __fadd_rn(v, part[w][r][t]);
    if (e0 + r < E) a.logits[(size_t)t * E + e0 + r] = v;
  }
  if (last_arrival(&a.cnt[0], (int)gridDim.x, &last_s)) route_tokens<PER>(a, 0, T, lrow, kGvWarps);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Tensor-core logits of a BM x 64 tile (tokens x experts).  Four warps as
// WM x WN; warp tile (16 MI) x (8 NI).  Shared memory per stage: BM rows of
// x then 64 rows of Wr, each kRtLd bf16 (144 bytes: ldmatrix rows fall in
// distinct bank groups).
template <int MI, int NI, int WM, int WN, int STAGES>
__global__ void __launch_bounds__(128) router_mma_kernel(RouterArgs a) {
  static_assert(WM * WN == 4 && 8 * NI * WN == 64, "four warps over 64 experts");
  constexpr int BM = 16 * MI * WM, BN = 64;
  constexpr int ROWS = BM + BN;
  extern __shared__ __align__(16) uint16_t rsm[];  // [STAGES][ROWS][kRtLd]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp / WN, wn = warp % WN;
  const int t0 = blockIdx.x * BM, e0 = blockIdx.y * BN;
  const int T = a.T, E = a.E, H = a.H;
  const int nk = H / kRtKc;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  auto load = [&](int kc, int st) {
    uint16_t *base = rsm + (size_t)st * ROWS * kRtLd;
    for (int v = tid; v < ROWS * 8; v += 128) {
      const int r = v >> 3, p = v & 7;
      const bool isx = r < BM;
      const int row = isx ? t0 + r : e0 + r - BM;
      const bool ok = row < (isx ? T : E);
      const uint16_t *src = (isx ? a.x : a.wr) + (size_t)(ok ? row : 0) * H + kc * kRtKc + 8 * p;
      cp_async_16z(base + r * kRtLd + 8 * p, src, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[MI][NI][4];
#pragma unroll
  for (int i = 0; i < MI; ++i)
#pragma unroll
    for (int j = 0; j < NI; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][j][q] = 0.f;
  // chunks 0 .. STAGES - 2 in flight; every iteration commits one group
  // (empty past the end), so "all but the newest STAGES - 1 groups done"
  // always means chunk kc has landed
#pragma unroll
  for (int c = 0; c < STAGES - 1; ++c) {
    if (c < nk) load(c, c);
    else asm volatile("cp.async.commit_group;" ::: "memory");
  }
  // ldmatrix lane addresses: A matrices (rows 0-7 | 8-15) x (k 0-7 | 8-15);
  // B matrices (n 0-7 | k 0-7), (n 0-7 | k 8-15), (n 8-15 | k 0-7), (n 8-15 | k 8-15)
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_col = (lane >> 4) * 8;
  const int b_row = (lane & 7) + (lane >> 4) * 8, b_col = ((lane >> 3) & 1) * 8;
  for (int kc = 0; kc < nk; ++kc) {
    const int st = kc % STAGES;
    if (kc + STAGES - 1 < nk) load(kc + STAGES - 1, (kc + STAGES - 1) % STAGES);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group %0;" ::"n"(STAGES - 1) : "memory");
    __syncthreads();
    const uint32_t sx = smem_u32(rsm + (size_t)st * ROWS * kRtLd);
    const uint32_t sw = sx + BM * kRtLd * 2;
#pragma unroll
    for (int kk = 0; kk < kRtKc; kk += 16) {
      uint32_t af[MI][4], bf[NI][2];
#pragma unroll
      for (int i = 0; i < MI; ++i)
        ldmatrix_x4(af[i], sx + ((16 * (MI * wm + i) + a_row) * kRtLd + kk + a_col) * 2);
#pragma unroll
      for (int j = 0; j < NI; j += 2) {
        uint32_t r[4];
        ldmatrix_x4(r, sw + ((8 * (NI * wn + j) + b_row) * kRtLd + kk + b_col) * 2);
        bf[j][0] = r[0];
        bf[j][1] = r[1];
        bf[j + 1][0] = r[2];
        bf[j + 1][1] = r[3];
      }
#pragma unroll
      for (int i = 0; i < MI; ++i)
#pragma unroll
        for (int j = 0; j < NI; ++j) mma_bf16_16816(acc[i][j], af[i], bf[j][0], bf[j][1]);
    }
    __syncthreads();  // this stage is free for the chunk STAGES - 1 ahead
  }
  // fragment (row gi / gi + 8, columns 2 t4, 2 t4 + 1) -> logits
  const int gi = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int i = 0; i < MI; ++i)
#pragma unroll
    for (int j = 0; j < NI; ++j) {
      const int t = t0 + 16 * (MI * wm + i) + gi, e = e0 + 8 * (NI * wn + j) + 2 * t4;
      if (e < E) {
        if (t < T) *reinterpret_cast<float2 *>(a.logits + (size_t)t * E + e) = make_float2(acc[i][j][0], acc[i][j][1]);
        if (t + 8 < T)
          *reinterpret_cast<float2 *>(a.logits + (size_t)(t + 8) * E + e) = make_float2(acc[i][j][2], acc[i][j][3]);
      }
    }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename Kern>
static moe_status router_launch(Kern kern, dim3 grid, dim3 block, size_t smem, const RouterArgs &a,
                                cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// the dynamic shared-memory opt-in of a kernel, set once per device; `done`
// is that kernel's own record (host threads may race here; the call is
// idempotent)
template <typename Kern>
static moe_status set_smem_once(Kern kern, size_t smem, std::atomic<unsigned long long> &done) {
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return MOE_OK;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  done.fetch_or(bit, std::memory_order_acq_rel);
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
  const bool small_e = E <= 256;
  if (T <= kGvMaxTok) {  // decode: every CTA reads two experts' rows once
    const dim3 grid((E + kGvRows - 1) / kGvRows), block(kGvWarps * 32);
    if (small_e) return router_launch(router_gemv_kernel<8>, grid, block, kGvWarps * 8 * 32 * 4, a, s);
    const size_t smem = kGvWarps * 32 * 32 * 4;
    static std::atomic<unsigned long long> done{0};
    const moe_status st = set_smem_once(router_gemv_kernel<32>, smem, done);
    return st != MOE_OK ? st : router_launch(router_gemv_kernel<32>, grid, block, smem, a, s);
  }
  // the GEMM, then the routing launch
  moe_status st;
  const int by = (E + 63) / 64;
  if (T >= 256) {
    constexpr int ST = 8, BM = 64;
    const size_t smem = (size_t)ST * (BM + 64) * kRtLd * 2;
    auto kern = router_mma_kernel<2, 4, 2, 2, ST>;
    static std::atomic<unsigned long long> done{0};
    st = set_smem_once(kern, smem, done);
    if (st == MOE_OK) st = router_launch(kern, dim3((T + BM - 1) / BM, by), dim3(128), smem, a, s);
  } else {
    constexpr int ST = 6, BM = 16;
    const size_t smem = (size_t)ST * (BM + 64) * kRtLd * 2;
    auto kern = router_mma_kernel<1, 2, 1, 4, ST>;
    static std::atomic<unsigned long long> done{0};
    st = set_smem_once(kern, smem, done);
    if (st == MOE_OK) st = router_launch(kern, dim3((T + BM - 1) / BM, by), dim3(128), smem, a, s);
  }
  if (st != MOE_OK) return st;
  return route_rows(a.logits, T, E, k, idx, w, s);
}
