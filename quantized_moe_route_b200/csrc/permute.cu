// permute.cu -- group the T*k routed rows by expert ("drama-rs", section
// "Apple Silicon (MLX)": prefill groups rows by routed expert).
//
// Stream-ordered kernels, no global atomics:
//   1. per-chunk expert histograms (shared-memory counters),
//   2. one block: totals, exclusive scan -> offsets, per-chunk bases,
//   3. per chunk: stable ranks with warp match + popc, scatter of
//      sorted_rows / inv,
//   4. optional: the gather of x rows into x_perm, one warp per destination
//      row, many rows in flight across the whole GPU.
#include <algorithm>

#include "common.cuh"

namespace moe {

constexpr int kPermChunk = 256;  // rows per chunk (one block each)

__global__ void perm_hist_kernel(const int32_t *__restrict__ idx, int R, int E,
                                 int32_t *__restrict__ hist) {
  grid_dep_wait();
  extern __shared__ int32_t sh[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh[e] = 0;
  __syncthreads();
  const int r0 = blockIdx.x * kPermChunk;
  for (int r = r0 + threadIdx.x; r < min(R, r0 + kPermChunk); r += blockDim.x)
    if ((unsigned)idx[r] < (unsigned)E) atomicAdd(&sh[idx[r]], 1);  // ids outside [0, E) are skipped
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = sh[e];
  grid_dep_trigger();
}

// One block of 1024 threads.  Each expert's chunks are split among S
// consecutive threads (S a power of two, S * E <= 1024 where E allows): every
// thread sums a contiguous range of chunks, the S partial sums are combined
// with warp shuffles (totals, then the per-chunk running bases).
__global__ void perm_scan_kernel(const int32_t *__restrict__ hist, int nchunks, int E, int S,
                                 int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                                 int32_t *__restrict__ base) {
  grid_dep_wait();
  extern __shared__ int32_t sh[];  // [E] totals then scanned
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int per = (nchunks + S - 1) / S;  // chunks of one thread
  const int ngroups = (E * S + blockDim.x - 1) / blockDim.x;
  for (int g = 0; g < ngroups; ++g) {
    const int idx = g * blockDim.x + threadIdx.x;
    const int e = idx / S, part = idx % S;
    int sum = 0;
    if (e < E)
      for (int c = part * per; c < min(nchunks, (part + 1) * per); ++c) sum += hist[(size_t)c * E + e];
    int tot = sum;
    for (int o = 1; o < S; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if (e < E && part == 0) {
      sh[e] = tot;
      counts[e] = tot;
    }
  }
  __syncthreads();
  // block-wide exclusive scan of sh[0..E), 1024 entries per pass
  __shared__ int32_t warp_sum[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    __syncthreads();
    const int e = e0 + threadIdx.x;
    const int v = e < E ? sh[e] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int ws = lane < (int)(blockDim.x >> 5) ? warp_sum[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += n;
      }
      warp_sum[lane] = ws;  // inclusive over warps
    }
    __syncthreads();
    const int excl = carry + (wid ? warp_sum[wid - 1] : 0) + incl - v;
    if (e < E) {
      sh[e] = excl;
      offsets[e] = excl;
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = excl + v;
  }
  __syncthreads();
  if (threadIdx.x == 0) offsets[E] = carry;
  // base[c][e] = offsets[e] + sum over c' < c of hist[c'][e]: each thread
  // starts its chunk range after the ranges of the lower parts
  for (int g = 0; g < ngroups; ++g) {
    const int idx = g * blockDim.x + threadIdx.x;
    const int e = idx / S, part = idx % S;
    const int c0 = part * per, c1 = min(nchunks, (part + 1) * per);
    int sum = 0;
    if (e < E)
      for (int c = c0; c < c1; ++c) sum += hist[(size_t)c * E + e];
    int incl = sum;  // inclusive scan over the S parts of this expert
    for (int o = 1; o < S; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (part >= o) incl += n;
    }
    if (e < E) {
      int run = sh[e] + incl - sum;
      for (int c = c0; c < c1; ++c) {
        base[(size_t)c * E + e] = run;
        run += hist[(size_t)c * E + e];
      }
    }
  }
  grid_dep_trigger();
}

// One warp assigns positions to the chunk's rows 32 at a time, in row order.
__global__ void perm_scatter_kernel(const int32_t *__restrict__ idx, int R, int E,
                                    const int32_t *__restrict__ base,
                                    int32_t *__restrict__ sorted_rows, int32_t *__restrict__ inv) {
  grid_dep_wait();
  extern __shared__ int32_t run[];  // [E] running position per expert
  const int r0 = blockIdx.x * kPermChunk;
  const int nrows = min(R - r0, kPermChunk);
  for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = base[(size_t)blockIdx.x * E + e];
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int ids[kPermChunk / 32];  // the chunk's expert ids, all loads issued up front
#pragma unroll
    for (int s8 = 0; s8 < kPermChunk / 32; ++s8) {
      const int i = 32 * s8 + lane;
      ids[s8] = i < nrows ? idx[r0 + i] : -1;
    }
#pragma unroll
    for (int s8 = 0; s8 < kPermChunk / 32; ++s8) {
      const int i0 = 32 * s8;
      if (i0 >= nrows) break;
      const int i = i0 + lane;
      const int ei = ids[s8];
      const bool valid = (unsigned)ei < (unsigned)E;  // ids outside [0, E) are skipped
      const int e = valid ? ei : -1 - lane;           // invalid lanes never match
      const uint32_t active = __ballot_sync(0xffffffffu, valid);
      const uint32_t peers = __match_any_sync(0xffffffffu, e) & active;
      if (valid) {
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int p = run[e] + rank;
        sorted_rows[p] = r0 + i;
        inv[r0 + i] = p;
      }
      __syncwarp();
      if (valid && lane == __ffs(peers) - 1) run[e] += __popc(peers);
      __syncwarp();
    }
  }
  grid_dep_trigger();
}

// x_perm[p] = x[sorted_rows[p] / k] for the offsets[E] grouped rows: warp w
// of the grid copies rows w, w + nwarps, ...; each lane moves up to eight
// 16-byte vectors of a row at once (all loads before the stores).
__global__ void perm_gather_kernel(const int32_t *__restrict__ sorted_rows,
                                   const int32_t *__restrict__ offsets, int E, int k,
                                   const uint16_t *__restrict__ x, int H,
                                   uint16_t *__restrict__ x_perm) {
  grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int nwarps = (int)(gridDim.x * blockDim.x) >> 5;
  const int total = offsets[E];
  const int vec = H / 8;  // 16-byte vectors per row
  for (int p = (int)(blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < total; p += nwarps) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)(sorted_rows[p] / k) * H);
    uint4 *dst = reinterpret_cast<uint4 *>(x_perm + (size_t)p * H);
    for (int v0 = 0; v0 < vec; v0 += 8 * 32) {
      uint4 buf[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = v0 + 32 * j + lane;
        if (v < vec) buf[j] = src[v];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = v0 + 32 * j + lane;
        if (v < vec) dst[v] = buf[j];
      }
    }
  }
  grid_dep_trigger();
}

}  // namespace moe

using namespace moe;

static int perm_chunks(int R) { return (R + kPermChunk - 1) / kPermChunk; }

extern "C" MOE_API size_t moe_permute_workspace_bytes(int T, int k, int E) {
  if (T <= 0 || k <= 0 || E <= 0) return 0;
  return 2 * sizeof(int32_t) * (size_t)perm_chunks(T * k) * (size_t)E;
}

extern "C" MOE_API moe_status moe_permute(const int32_t *idx, int T, int k, int E,
                                          const uint16_t *x, int H, int32_t *counts,
                                          int32_t *offsets, int32_t *sorted_rows, int32_t *inv,
                                          uint16_t *x_perm, void *ws, size_t ws_bytes,
                                          moe_stream_t stream) {
  if (T < 0 || k <= 0 || E <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > 8192) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (T == 0) {  // empty batch: all counts zero, offsets all zero
    cudaError_t e1 = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s);
    cudaError_t e2 = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
    if (e1 != cudaSuccess || e2 != cudaSuccess) {
      set_cuda_error(e1 != cudaSuccess ? e1 : e2);
      return MOE_ERR_CUDA;
    }
    return MOE_OK;
  }
  if (!idx || !sorted_rows || !inv) return MOE_ERR_INVALID_ARG;
  const bool gather = (x_perm != nullptr);
  if (gather && (!x || H <= 0)) return MOE_ERR_INVALID_ARG;
  if (gather && (H % 8 || reinterpret_cast<uintptr_t>(x) % 16 ||
                 reinterpret_cast<uintptr_t>(x_perm) % 16))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * k > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int R = T * k, nch = perm_chunks(R);
  if (!ws || ws_bytes < moe_permute_workspace_bytes(T, k, E)) return MOE_ERR_WORKSPACE;
  int32_t *hist = static_cast<int32_t *>(ws);
  int32_t *base = hist + (size_t)nch * E;
  const size_t shE = sizeof(int32_t) * (size_t)E;
  moe_status st = launch_pdl(perm_hist_kernel, dim3(nch), dim3(256), shE, s, idx, R, E, hist);
  if (st != MOE_OK) return st;
  int S = 1;  // threads per expert in the scan: a power of two, S * E <= 1024, S <= 32
  while (S < 32 && 2 * S * E <= 1024 && S < nch) S *= 2;
  st = launch_pdl(perm_scan_kernel, dim3(1), dim3(1024), shE, s, hist, nch, E, S, counts, offsets, base);
  if (st != MOE_OK) return st;
  st = launch_pdl(perm_scatter_kernel, dim3(nch), dim3(256), shE, s, idx, R, E, (const int32_t *)base,
                  sorted_rows, inv);
  if (st != MOE_OK || !gather) return st;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int blocks = (int)std::min<long long>((R + 7) / 8, 8LL * nsm);  // 8 warps per block
  return launch_pdl(perm_gather_kernel, dim3(blocks), dim3(256), 0, s, (const int32_t *)sorted_rows,
                    (const int32_t *)offsets, E, k, x, H, x_perm);
}
