// decode.cu -- weight-streaming expert FFN for small batches (1..16 tokens).
//
// Decode is memory-bandwidth bound ("drama-rs", section "Experts: where they
// run"; each decode step streams its GEMV weights, section "Footprint and
// speed").  This kernel reads every selected expert's packed int4 weights
// from HBM exactly once per call, whatever the number of tokens routed to it.
//
// Work items (static round-robin over a persistent grid, all CTAs resident):
//   A(u, p): expert slot u, 16 features p: the gate strip and the up strip of
//            those features (contiguous in the packed layout), all H inputs;
//            g, u, h = SiLU(g) * u in registers; h -> workspace; flag[u] += 1.
//   B(u, c): expert slot u, 64 outputs c: four down strips, all F inputs;
//            waits (bounded) until flag[u] == F/16, then y_rows.
// Every A item precedes every B item in the global order, and a CTA runs its
// items in increasing order, so the lowest unfinished item never waits.
//
// Arithmetic: a packed 32-bit word holds the eight 4-bit codes one lane needs
// for one m16n8k16 A fragment; OR-ing 0x4300 into each 16-bit half turns code
// q into the bf16 value 128 + q exactly.  The tensor core then forms
// D = sum (128 + q) x in fp32 for one 64-channel group, and the group's affine
// map is applied once per output and token:
//   sum_k (q s + m) x_k = s D + (m - 128 s) X,   X = sum_k x_k.
// Activations enter as bf16 (exact), h is rounded to bf16 for the down
// projection; all sums are fp32.
#include "common.cuh"

namespace moe {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecMaxTok = 16;   // tokens per expert per call (two n8 blocks)
constexpr int kDecMaxRows = 256; // T * k
constexpr int kDecMaxE = 1024;
constexpr int kDecOutRows = 64;  // outputs per B item (4 strips)

struct DecodeArgs {
  const uint8_t *gu;
  const uint8_t *dn;
  size_t gu_stride, dn_stride;  // bytes per expert
  const uint16_t *x;
  const int32_t *idx;
  float *y_rows;
  float *hbuf;  // [T*k][F]
  int *flags;   // [kDecMaxRows] per-slot counters, [kDecMaxRows] CTA-done counter
  int *err;
  int T, k, E, H, F;
  int nstages;
  uint32_t stage_bytes;
};

struct DecodeSmem {
  // offsets (bytes) into dynamic shared memory
  uint32_t x, xsum, stages, red, h, hsum, bars, meta, total;
};

__host__ __device__ inline DecodeSmem decode_smem_layout(int T, int H, int F, int nstages,
                                                         uint32_t stage_bytes) {
  DecodeSmem L;
  uint32_t o = 0;
  auto take = [&](uint32_t bytes, uint32_t align) {
    o = (o + align - 1) / align * align;
    uint32_t at = o;
    o += bytes;
    return at;
  };
  L.stages = take((uint32_t)nstages * stage_bytes, 128);
  L.x = take((uint32_t)T * H * 2, 16);
  L.xsum = take((uint32_t)T * (H / 64) * 4, 16);
  L.red = take(kDecWarps * 2 * 16 * kDecMaxTok * 4, 16);
  L.h = take((uint32_t)kDecMaxTok * F * 2, 16);
  L.hsum = take((uint32_t)kDecMaxTok * (F / 64) * 4, 16);
  L.bars = take((uint32_t)nstages * 8, 8);
  // meta: flag/slot_of [E], slot_cnt [256], slot_off [257], slot_rows [256], ridx [256], misc
  L.meta = take((kDecMaxE + 4 * kDecMaxRows + 8) * 4, 16);
  L.total = o;
  return L;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Exclusive scan over blockDim (256) values; returns the exclusive prefix and
// the total through *total.
__device__ int block_exclusive_scan(int v, int *wsum, int *total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int s = lane < kDecWarps ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    if (lane < kDecWarps) wsum[lane] = s;
  }
  __syncthreads();
  int ex = (wid ? wsum[wid - 1] : 0) + incl - v;
  *total = wsum[kDecWarps - 1];
  __syncthreads();
  return ex;
}

// Build the 4 A-fragment registers of one k16 step from one packed word.
__device__ __forceinline__ void w4_frag(uint32_t w, uint32_t a[4]) {
  a[0] = (w & 0x000F000Fu) | 0x43004300u;
  a[1] = ((w >> 4) & 0x000F000Fu) | 0x43004300u;
  a[2] = ((w >> 8) & 0x000F000Fu) | 0x43004300u;
  a[3] = ((w >> 12) & 0x000F000Fu) | 0x43004300u;
}

// One warp, one 16x64 block of one matrix against up to 16 activation rows
// held in shared memory as bf16 [n][ld]: accumulates the folded group result
// into acc[nb][4].
template <int NB>
__device__ __forceinline__ void block_mma(const uint8_t *blk, const uint16_t *act, int ld,
                                          int kbase, const int *tok_of, int ntok,
                                          const float *gsum, int gsum_ld, int gidx,
                                          float acc[2][4]) {
  const int lane = threadIdx.x & 31, gi = lane >> 2, t4 = lane & 3;
  const uint4 cw = *reinterpret_cast<const uint4 *>(blk + 16 * lane);
  const uint32_t sm_lo = *reinterpret_cast<const uint32_t *>(blk + kBlkCodeBytes + 4 * gi);
  const uint32_t sm_hi = *reinterpret_cast<const uint32_t *>(blk + kBlkCodeBytes + 4 * (gi + 8));
  const float s0 = f16_bits_to_f32((uint16_t)(sm_lo & 0xFFFFu));
  const float m0 = f16_bits_to_f32((uint16_t)(sm_lo >> 16));
  const float s1 = f16_bits_to_f32((uint16_t)(sm_hi & 0xFFFFu));
  const float m1 = f16_bits_to_f32((uint16_t)(sm_hi >> 16));
  const float c0 = __fmaf_rn(-128.f, s0, m0), c1 = __fmaf_rn(-128.f, s1, m1);
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int n = nb * 8 + gi;  // this lane's B column (token slot)
    const bool live = n < ntok;
    const uint16_t *arow = act + (size_t)(live ? tok_of[n] : 0) * ld + kbase + 2 * t4;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t a[4];
      w4_frag(words[j], a);
      uint32_t b0 = live ? *reinterpret_cast<const uint32_t *>(arow + 16 * j) : 0u;
      uint32_t b1 = live ? *reinterpret_cast<const uint32_t *>(arow + 16 * j + 8) : 0u;
      mma_bf16_16816(d, a, b0, b1);
    }
    // columns of this lane's D fragment: tokens nb*8 + 2*t4 (+1)
    const int na = nb * 8 + 2 * t4, nbb = na + 1;
    const float xa = na < ntok ? gsum[(size_t)tok_of[na] * gsum_ld + gidx] : 0.f;
    const float xb = nbb < ntok ? gsum[(size_t)tok_of[nbb] * gsum_ld + gidx] : 0.f;
    acc[nb][0] += __fmaf_rn(s0, d[0], c0 * xa);
    acc[nb][1] += __fmaf_rn(s0, d[1], c0 * xb);
    acc[nb][2] += __fmaf_rn(s1, d[2], c1 * xa);
    acc[nb][3] += __fmaf_rn(s1, d[3], c1 * xb);
  }
}

// Scatter a warp's D-fragment accumulators into red[warp][row][token].
__device__ __forceinline__ void frag_to_red(float *red, const float acc[2][4], int nbmax) {
  const int lane = threadIdx.x & 31, gi = lane >> 2, t4 = lane & 3;
  for (int nb = 0; nb < nbmax; ++nb) {
    const int n = nb * 8 + 2 * t4;
    red[gi * kDecMaxTok + n] = acc[nb][0];
    red[gi * kDecMaxTok + n + 1] = acc[nb][1];
    red[(gi + 8) * kDecMaxTok + n] = acc[nb][2];
    red[(gi + 8) * kDecMaxTok + n + 1] = acc[nb][3];
  }
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const DecodeSmem L = decode_smem_layout(a.T, a.H, a.F, a.nstages, a.stage_bytes);
  uint16_t *x_s = reinterpret_cast<uint16_t *>(smem + L.x);
  float *xsum_s = reinterpret_cast<float *>(smem + L.xsum);
  float *red_s = reinterpret_cast<float *>(smem + L.red);
  uint16_t *h_s = reinterpret_cast<uint16_t *>(smem + L.h);
  float *hsum_s = reinterpret_cast<float *>(smem + L.hsum);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  int *meta = reinterpret_cast<int *>(smem + L.meta);
  int *slot_of = meta;                          // [E]
  int *slot_cnt = slot_of + kDecMaxE;           // [256]
  int *slot_off = slot_cnt + kDecMaxRows;       // [257]
  int *slot_rows = slot_off + kDecMaxRows + 1;  // [256]
  int *ridx = slot_rows + kDecMaxRows;          // [256]
  int *misc = ridx + kDecMaxRows;               // [0] U, [1] abort, [2..] scan scratch
  __shared__ int wsum[kDecWarps];
  __shared__ int tok_list[kDecMaxTok];
  __shared__ int ident[kDecMaxTok];

  const int tid = threadIdx.x, warp = tid >> 5;
  const int T = a.T, k = a.k, E = a.E, H = a.H, F = a.F;
  const int R = T * k, Gh = H / 64, Gf = F / 64;
  const uint32_t stripA = (uint32_t)Gh * kBlkBytes, stripB = (uint32_t)Gf * kBlkBytes;

  if (tid == 0) {
    for (int s = 0; s < a.nstages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  pdl_wait();  // inputs of this call may come from the previous kernel

  // ---- routing table: unique experts (ascending id) and their rows
  for (int e = tid; e < E; e += kDecThreads) slot_of[e] = 0;
  __syncthreads();
  if (tid < R) {
    int e = a.idx[tid];
    e = (e < 0 || e >= E) ? 0 : e;  // out-of-range ids are outside the contract; keep memory safe
    ridx[tid] = e;
    slot_of[e] = 1;
  }
  __syncthreads();
  {
    const int per = (E + kDecThreads - 1) / kDecThreads;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      int e = tid * per + i;
      if (e < E) local += slot_of[e];
    }
    int total;
    int ex = block_exclusive_scan(local, wsum, &total);
    for (int i = 0; i < per; ++i) {
      int e = tid * per + i;
      if (e < E) {
        int f = slot_of[e];
        slot_of[e] = f ? ex : -1;
        ex += f;
      }
    }
    if (tid == 0) misc[0] = total, misc[1] = 0;
  }
  if (tid < kDecMaxRows) slot_cnt[tid] = 0;
  if (tid < kDecMaxTok) ident[tid] = tid;
  __syncthreads();
  const int U = misc[0];
  int my_slot = -1, my_rank = 0;
  if (tid < R) {
    const int e = ridx[tid];
    my_slot = slot_of[e];
    for (int r = 0; r < tid; ++r) my_rank += (ridx[r] == e);
    atomicAdd(&slot_cnt[my_slot], 1);
  }
  __syncthreads();
  {
    int v = tid < U ? slot_cnt[tid] : 0, total;
    int ex = block_exclusive_scan(v, wsum, &total);
    if (tid < U) slot_off[tid] = ex;
    if (tid == 0) slot_off[U] = total;
  }
  __syncthreads();
  if (tid < R) slot_rows[slot_off[my_slot] + my_rank] = tid;

  // ---- activations into shared memory (bf16) and their 64-channel sums
  {
    const int vec = T * H / 8;
    for (int v = tid; v < vec; v += kDecThreads)
      reinterpret_cast<uint4 *>(x_s)[v] = reinterpret_cast<const uint4 *>(a.x)[v];
  }
  __syncthreads();
  for (int q = tid; q < T * Gh; q += kDecThreads) {
    const int t = q / Gh, g = q % Gh;
    const uint16_t *xr = x_s + (size_t)t * H + 64 * g;
    float s = 0.f;
    for (int i = 0; i < 64; ++i) s += bf16_bits_to_f32(xr[i]);
    xsum_s[t * Gh + g] = s;
  }

  // ---- items of this CTA
  const int nA = U * (F / 16), nB = U * (H / kDecOutRows), nItems = nA + nB;
  const int G = gridDim.x;
  auto item_src = [&](int item, const uint8_t **src, uint32_t *bytes, int *slot, int *sub,
                      bool *isA) {
    if (item < nA) {
      *isA = true;
      *slot = item / (F / 16);
      *sub = item % (F / 16);
    } else {
      *isA = false;
      *slot = (item - nA) / (H / kDecOutRows);
      *sub = (item - nA) % (H / kDecOutRows);
    }
    const int e = ridx[slot_rows[slot_off[*slot]]];
    if (*isA) {
      *src = a.gu + (size_t)e * a.gu_stride + (size_t)(2 * *sub) * stripA;
      *bytes = 2 * stripA;
    } else {
      *src = a.dn + (size_t)e * a.dn_stride + (size_t)(4 * *sub) * stripB;
      *bytes = 4 * stripB;
    }
  };
  const int myCount = (blockIdx.x < nItems) ? (nItems - 1 - blockIdx.x) / G + 1 : 0;
  const uint64_t pol = policy_evict_first();
  __syncthreads();
  if (tid == 0) {
    for (int q = 0; q < min(myCount, a.nstages); ++q) {
      const uint8_t *src;
      uint32_t bytes;
      int slot, sub;
      bool isA;
      item_src(blockIdx.x + q * G, &src, &bytes, &slot, &sub, &isA);
      mbar_arrive_expect_tx(&bars[q], bytes);
      bulk_g2s_evict_first(smem + L.stages + (size_t)q * a.stage_bytes, src, bytes, &bars[q], pol);
    }
  }
  pdl_launch_dependents();

  for (int q = 0; q < myCount; ++q) {
    const int item = blockIdx.x + q * G;
    const int stage = q % a.nstages;
    const uint32_t parity = (uint32_t)(q / a.nstages) & 1u;
    const uint8_t *src;
    uint32_t bytes;
    int slot, sub;
    bool isA;
    item_src(item, &src, &bytes, &slot, &sub, &isA);
    const int r0 = slot_off[slot], ntok = slot_off[slot + 1] - r0;
    if (tid < kDecMaxTok) tok_list[tid] = tid < ntok ? slot_rows[r0 + tid] / k : 0;

    if (!isA) {  // B item: wait for every A item of this slot (bounded)
      if (tid == 0) {
        const int need = F / 16;
        uint32_t spins = 0;
        while (ld_acquire_gpu(&a.flags[slot]) < need) {
          if (++spins > (1u << 22)) {  // ~seconds: only a broken contract gets here
            atomicExch(a.err, DEVERR_DECODE_H_WAIT);
            misc[1] = 1;
            break;
          }
          __nanosleep(128);
        }
      }
      __syncthreads();
      if (misc[1]) break;
      // h of this slot's rows -> bf16 shared tile, and 64-channel sums
      for (int v = tid; v < ntok * F; v += kDecThreads) {
        const int n = v / F, f = v % F;
        const float hv = __ldcg(a.hbuf + (size_t)slot_rows[r0 + n] * F + f);
        h_s[n * F + f] = f32_to_bf16_bits(hv);
      }
      __syncthreads();
      for (int v = tid; v < ntok * Gf; v += kDecThreads) {
        const int n = v / Gf, g = v % Gf;
        float s = 0.f;
        for (int i = 0; i < 64; ++i) s += bf16_bits_to_f32(h_s[n * F + 64 * g + i]);
        hsum_s[n * Gf + g] = s;
      }
    }
    __syncthreads();

    // wait for this item's weights (every thread observes the barrier)
    const bool landed = mbar_wait_bounded(&bars[stage], parity, 1u << 26);
    if (__syncthreads_or(!landed)) {  // only a copy stalled for seconds gets here
      if (tid == 0) {
        atomicExch(a.err, DEVERR_DECODE_H_WAIT);
        misc[1] = 1;
      }
      break;
    }
    const uint8_t *st = smem + L.stages + (size_t)stage * a.stage_bytes;
    float acc0[2][4] = {}, acc1[2][4] = {};
    const int nbmax = ntok > 8 ? 2 : 1;
    if (isA) {
      for (int g = warp; g < Gh; g += kDecWarps) {
        if (nbmax == 2) {
          block_mma<2>(st + (size_t)g * kBlkBytes, x_s, H, 64 * g, tok_list, ntok, xsum_s, Gh, g, acc0);
          block_mma<2>(st + stripA + (size_t)g * kBlkBytes, x_s, H, 64 * g, tok_list, ntok, xsum_s, Gh, g, acc1);
        } else {
          block_mma<1>(st + (size_t)g * kBlkBytes, x_s, H, 64 * g, tok_list, ntok, xsum_s, Gh, g, acc0);
          block_mma<1>(st + stripA + (size_t)g * kBlkBytes, x_s, H, 64 * g, tok_list, ntok, xsum_s, Gh, g, acc1);
        }
      }
      frag_to_red(red_s + (size_t)(warp * 2 + 0) * 16 * kDecMaxTok, acc0, nbmax);
      frag_to_red(red_s + (size_t)(warp * 2 + 1) * 16 * kDecMaxTok, acc1, nbmax);
    } else {
      // warp -> strip (warp & 3), groups of parity (warp >> 2)
      const int strip = warp & 3;
      for (int g = warp >> 2; g < Gf; g += 2) {
        const uint8_t *blk = st + (size_t)strip * stripB + (size_t)g * kBlkBytes;
        // h_s rows are indexed by the slot position n itself
        if (nbmax == 2)
          block_mma<2>(blk, h_s, F, 64 * g, ident, ntok, hsum_s, Gf, g, acc0);
        else
          block_mma<1>(blk, h_s, F, 64 * g, ident, ntok, hsum_s, Gf, g, acc0);
      }
      frag_to_red(red_s + (size_t)warp * 16 * kDecMaxTok, acc0, nbmax);
    }
    __syncthreads();
    // the stage is free again: refill it with item q + nstages
    if (tid == 0 && q + a.nstages < myCount) {
      const uint8_t *nsrc;
      uint32_t nbytes;
      int ns, nsub;
      bool nA2;
      item_src(blockIdx.x + (q + a.nstages) * G, &nsrc, &nbytes, &ns, &nsub, &nA2);
      mbar_arrive_expect_tx(&bars[stage], nbytes);
      bulk_g2s_evict_first(smem + L.stages + (size_t)stage * a.stage_bytes, nsrc, nbytes,
                           &bars[stage], pol);
    }
    if (isA) {
      // reduce over warps: thread -> (row, token)
      const int row = tid >> 4, n = tid & 15;
      if (n < ntok) {
        float g = 0.f, u = 0.f;
        for (int w = 0; w < kDecWarps; ++w) {
          g += red_s[(size_t)(w * 2 + 0) * 16 * kDecMaxTok + row * kDecMaxTok + n];
          u += red_s[(size_t)(w * 2 + 1) * 16 * kDecMaxTok + row * kDecMaxTok + n];
        }
        const float h = g / (1.0f + expf(-g)) * u;
        a.hbuf[(size_t)slot_rows[r0 + n] * F + 16 * sub + row] = h;
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) red_release_gpu_add(&a.flags[slot], 1);
    } else {
      for (int v = tid; v < 4 * 16 * kDecMaxTok; v += kDecThreads) {
        const int strip = v / (16 * kDecMaxTok), rem = v % (16 * kDecMaxTok);
        const int row = rem / kDecMaxTok, n = rem % kDecMaxTok;
        if (n < ntok) {
          float y = red_s[(size_t)strip * 16 * kDecMaxTok + rem] +
                    red_s[(size_t)(strip + 4) * 16 * kDecMaxTok + rem];
          a.y_rows[(size_t)slot_rows[r0 + n] * H + kDecOutRows * sub + 16 * strip + row] = y;
        }
      }
    }
    __syncthreads();
  }

  // ---- aborted: let in-flight copies land before the CTA exits
  if (misc[1] && tid == 0) {
    for (int s = 0; s < a.nstages; ++s) mbar_wait_bounded(&bars[s], 0, 1u << 20);
  }
  // ---- last CTA out resets the slot counters for the next call
  if (tid == 0) {
    __threadfence();
    int done = atomicAdd(&a.flags[kDecMaxRows], 1);
    if (done == (int)gridDim.x - 1) {
      for (int s = 0; s < kDecMaxRows; ++s) a.flags[s] = 0;
      a.flags[kDecMaxRows] = 0;
      __threadfence();
    }
  }
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_decode_workspace_bytes(int T, int k, int F) {
  if (T <= 0 || k <= 0 || F <= 0) return 0;
  return 4096 + sizeof(float) * (size_t)T * k * F;
}

extern "C" MOE_API moe_status moe_ffn_w4a16_decode(const moe_w4_layer *layer, const uint16_t *x,
                                                   const int32_t *idx, int T, int k, float *y_rows,
                                                   void *ws, size_t ws_bytes,
                                                   moe_stream_t stream) {
  if (!layer || T < 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  const int E = layer->E, H = layer->H, F = layer->F;
  if (E <= 0 || H <= 0 || F <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (H % 64 || F % 64 || E > kDecMaxE || T > kDecMaxTok || T * k > kDecMaxRows)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!layer->gate_up || !layer->down || !x || !idx || !y_rows) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(layer->gate_up) % 16 ||
      reinterpret_cast<uintptr_t>(layer->down) % 16 || reinterpret_cast<uintptr_t>(x) % 16)
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_decode_workspace_bytes(T, k, F)) return MOE_ERR_WORKSPACE;

  DecodeArgs a;
  a.gu = static_cast<const uint8_t *>(layer->gate_up);
  a.dn = static_cast<const uint8_t *>(layer->down);
  a.gu_stride = w4_packed_bytes(2 * F, H);
  a.dn_stride = w4_packed_bytes(H, F);
  a.x = x;
  a.idx = idx;
  a.y_rows = y_rows;
  a.flags = static_cast<int *>(ws);
  a.hbuf = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + 4096);
  a.err = device_error_word();
  if (!a.err) return MOE_ERR_CUDA;
  a.T = T;
  a.k = k;
  a.E = E;
  a.H = H;
  a.F = F;
  const uint32_t itemA = 2u * (H / 64) * kBlkBytes, itemB = 4u * (F / 64) * kBlkBytes;
  a.stage_bytes = (max(itemA, itemB) + 127u) / 128u * 128u;

  int dev = 0, sms = 0, smem_max = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  int nst = 8;
  while (nst > 1 && decode_smem_layout(T, H, F, nst, a.stage_bytes).total > (uint32_t)smem_max - 1024)
    --nst;
  const DecodeSmem L = decode_smem_layout(T, H, F, nst, a.stage_bytes);
  if (L.total > (uint32_t)smem_max - 1024) return MOE_ERR_UNSUPPORTED_SHAPE;
  a.nstages = nst;
  static bool attr_done[64] = {false};
  if (dev < 64 && !attr_done[dev]) {
    cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max - 1024);
    attr_done[dev] = true;
  }
  // Upper bound on items: the grid never exceeds the SM count (one CTA per
  // SM, all resident, as the cross-CTA waits require).
  const int maxItems = T * k * (F / 16 + H / kDecOutRows);
  const int grid = max(1, min(sms, maxItems));

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = as_stream(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel, a);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the decode call.
//
// Some callers cannot allocate device memory at all: plugins and embedded
// hosts whose device memory is owned and budgeted by the host application,
// and programs with a fixed memory plan that forbids any allocation once they
// have started serving.  They cannot supply the scratch workspace that
// moe_ffn_w4a16_decode needs, so this variant keeps its scratch (the per-slot
// counters and the h buffer) in one fixed array in the library's own device
// memory instead.  The array is a module global: every GPU that loads the
// library holds it until the process exits.
// ---------------------------------------------------------------------------
namespace moe {

constexpr size_t kStaticFlagBytes = 4096;
constexpr size_t kStaticHBytes = 512 * 1024;  // T*k*F*4 bytes of h at most
constexpr size_t kStaticScratchBytes = kStaticFlagBytes + kStaticHBytes;

static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device, looked up once per
// device (the lookup needs that device to be current).
static uint8_t *static_scratch_address(moe_status *st) {
  static uint8_t *addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    set_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
    *st = MOE_ERR_CUDA;
    return nullptr;
  }
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      set_cuda_error(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
      *st = MOE_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = static_cast<uint8_t *>(p);
  }
  *st = MOE_OK;
  return addr[dev];
}

}  // namespace moe

extern "C" MOE_API moe_status moe_ffn_w4a16_decode_static(const moe_w4_layer *layer,
                                                          const uint16_t *x, const int32_t *idx,
                                                          int T, int k, float *y_rows,
                                                          moe_stream_t stream) {
  if (!layer || T < 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  const int E = layer->E, H = layer->H, F = layer->F;
  if (E <= 0 || H <= 0 || F <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (H % 64 || F % 64 || E > kDecMaxE || T > kDecMaxTok || T * k > kDecMaxRows)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  // the fixed scratch holds h for at most kStaticHBytes / 4 values
  if ((size_t)T * k * F * sizeof(float) > kStaticHBytes) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  if (!layer->gate_up || !layer->down || !x || !idx || !y_rows) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(layer->gate_up) % 16 ||
      reinterpret_cast<uintptr_t>(layer->down) % 16 || reinterpret_cast<uintptr_t>(x) % 16)
    return MOE_ERR_INVALID_ARG;

  moe_status st;
  uint8_t *scratch = static_scratch_address(&st);
  if (!scratch) return st;
  int *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  // The array keeps whatever the previous call left in it; the counters must
  // start at zero, so clear them on the caller's stream before the launch.
  cudaError_t e = cudaMemsetAsync(scratch, 0, kStaticFlagBytes, as_stream(stream));
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }

  DecodeArgs a;
  a.gu = static_cast<const uint8_t *>(layer->gate_up);
  a.dn = static_cast<const uint8_t *>(layer->down);
  a.gu_stride = w4_packed_bytes(2 * F, H);
  a.dn_stride = w4_packed_bytes(H, F);
  a.x = x;
  a.idx = idx;
  a.y_rows = y_rows;
  a.flags = reinterpret_cast<int *>(scratch);
  a.hbuf = reinterpret_cast<float *>(scratch + kStaticFlagBytes);
  a.err = err;
  a.T = T;
  a.k = k;
  a.E = E;
  a.H = H;
  a.F = F;
  const uint32_t itemA = 2u * (H / 64) * kBlkBytes, itemB = 4u * (F / 64) * kBlkBytes;
  a.stage_bytes = (max(itemA, itemB) + 127u) / 128u * 128u;

  int dev = 0, sms = 0, smem_max = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  int nst = 8;
  while (nst > 1 && decode_smem_layout(T, H, F, nst, a.stage_bytes).total > (uint32_t)smem_max - 1024)
    --nst;
  const DecodeSmem L = decode_smem_layout(T, H, F, nst, a.stage_bytes);
  if (L.total > (uint32_t)smem_max - 1024) return MOE_ERR_UNSUPPORTED_SHAPE;
  a.nstages = nst;
  e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_max - 1024);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  const int maxItems = T * k * (F / 16 + H / kDecOutRows);
  const int grid = max(1, min(sms, maxItems));
  decode_kernel<<<grid, kDecThreads, L.total, as_stream(stream)>>>(a);
  return launch_status();
}
