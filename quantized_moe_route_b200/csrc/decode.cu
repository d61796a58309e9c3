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
//            g, u, h = SiLU(g) * u in registers; h -> workspace.
//   B(u, c): expert slot u, 64 outputs c: four down strips, all F inputs;
//            needs every h of slot u, then writes y_rows.
// Every A item precedes every B item in the global order and a CTA runs its
// items in increasing order, so the lowest unfinished item never waits.
//
// h handoff without fences: each h value travels as one 8-byte word
// {bf16 h, call epoch}; a B item polls the words of its slot until all carry
// this call's epoch (single-copy atomic 8-byte stores and loads), so no
// release fence or counter sits on the gate/up critical path.
//
// Arithmetic: a packed 32-bit word holds the eight 4-bit codes one lane needs
// for one m16n8k16 A fragment; OR-ing 0x4300 into each 16-bit half turns code
// q into the bf16 value 128 + q exactly.  The tensor core forms
// D = sum (128 + q) x in fp32 for one 64-channel group, and the group's affine
// map is applied once per output and token:
//   sum_k (q s + m) x_k = s D + (m - 128 s) X,   X = sum_k x_k.
// Activations enter as bf16 (exact), h is rounded to bf16 for the down
// projection; all sums are fp32.
//
// NVFP4 weights ("Drama 3 - NVFP4 routed experts", section "Quantization")
// use the same items and strip sizes (4.5 bits per weight).  Each token's x
// and each row's h are quantised to NVFP4 inside the kernel (per-row global,
// E4M3 scale per 16 channels, E2M1 codes) and held in shared memory as the
// exact f16 values E2M1 * S_b.  A code word gives two f16 fragment halves by
// moving the 3 magnitude bits to bits 9..11 and the sign to bit 15, which is
// the E2M1 value times 2^-14 for every code (0.5 lands on the f16 subnormal
// 2^-15); the tensor core sums one 16-channel block per m16n8k16 step, the
// weight block scale is applied to that step's result in fp32, and 2^14 and
// the two globals are applied once per output.
#include <atomic>

#include "decode_common.cuh"
#include "decode_items.cuh"
#include "route.cuh"

namespace moe {

struct DecodeArgs {
  const float *logits;       // fused form: router logits [T][E] (unless wr)
  const uint16_t *wr;        // fused int4 form, optional: bf16 router weights [E - shared][H];
                             // the kernel computes the logits
  unsigned long long *lbuf;  // with wr: [T][E - shared] words {fp32 logit, epoch}
  float *logits_out;         // with wr, optional: the computed logits fp32 [T][E - shared]
  uint16_t *y;               // fused form: combined bf16 output [T][H]
  int32_t *idx_out;          // fused form, optional: routing of every token
  float *w_out;
  unsigned long long *ybuf;  // fused form: [T*k][H] words {fp32 row output, epoch}
  const uint8_t *gu;
  const uint8_t *dn;
  size_t gu_stride, dn_stride;  // bytes per expert
  const float *g_gu, *g_d;      // NVFP4: per-expert global scales
  const uint16_t *x;
  const int32_t *idx;
  float *y_rows;
  unsigned long long *hbuf;  // [T*k][F] words {h << 32 | epoch}: bf16 h (int4), fp32 h (NVFP4)
  unsigned int *ctrl;        // [0] last epoch, [1] CTAs done
  int *err;
  int T, k, E, H, F;
  int nstages;               // even: team t owns the stages s = t (mod 2)
  uint32_t stage_bytes;
  uint32_t h_off;            // offset of a B item's h tile inside its stage
  uint32_t h_polls;          // bound of a B item's wait for h (polls of >= 100 ns)
  int starve_gate_up;        // test hook: A items write no h, so B items time out
  int shared;                // fused form: 1 = the layer's last expert is a shared expert
                             // (row k - 1 of every token, weight 1); routing scores E - 1
};

struct DecodeSmem {
  // byte offsets into dynamic shared memory
  uint32_t stages, x, xsum, hsum, bars, rbars, meta, total;
};


// Stage buffer: an A item's weights, or a B item's weights followed by its h
// tile; after the compute the same buffer holds the cross-warp partial sums.
__host__ __device__ inline uint32_t dec_stage_bytes(int T, int H, int F, uint32_t *h_off) {
  const uint32_t itemA = 2u * (H / 64) * kBlkBytes, itemB = 4u * (F / 64) * kBlkBytes;
  const uint32_t hoff = (itemB + 127u) / 128u * 128u;
  const uint32_t red = kTeamWarps * 2u * 16u * (uint32_t)dec_ntok_cols(T) * 4u;
  uint32_t b = itemA > hoff + (uint32_t)T * F * 2u ? itemA : hoff + (uint32_t)T * F * 2u;
  b = b > red ? b : red;
  *h_off = hoff;
  return (b + 127u) / 128u * 128u;
}

__host__ __device__ inline DecodeSmem decode_smem_layout(int fmt, int T, int H, int F, int nstages,
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
  // int4: 64-channel group sums of x and of each team's h;
  // NVFP4: the row globals of x and of each team's h
  // NVFP4: the row globals of x and of each team's h, each followed by the
  // rows' maxima (as bits)
  L.xsum = take(fmt == kFmtW4 ? (uint32_t)T * (H / 64) * 4 : 2u * T * 4, 16);
  L.hsum = take(fmt == kFmtW4 ? 2u * T * (F / 64) * 4 : 2u * 2u * T * 4, 16);
  L.bars = take((uint32_t)nstages * 8, 8);
  L.rbars = take(kDecWarps * 8, 8);  // router-row copies, one barrier per warp
  L.meta = take(3600 * 4, 16);  // routing tables + 256 x 8 row-set words
  L.total = o;
  return L;
}

// kFused = false: routing comes in (idx), the k rows of every token go out as
// fp32 y_rows.  kFused = true: the kernel routes the tokens itself from their
// logits (PER logits per lane) and writes the router-weighted combine y; each
// 64-output chunk of a token is combined by the down item of that token's
// highest expert slot, which waits only on lower-numbered items.
template <int kFmt, bool kFused, int PER>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(DecodeArgs a) {
  static_assert(kFmt == kFmtW4 || kFused, "the NVFP4 decode exists in the fused form only");
  constexpr bool kFp4 = kFmt == kFmtNvfp4;
  extern __shared__ __align__(128) uint8_t smem[];
  const DecodeSmem L = decode_smem_layout(kFmt, a.T, a.H, a.F, a.nstages, a.stage_bytes);
  uint16_t *x_s = reinterpret_cast<uint16_t *>(smem + L.x);
  float *xsum_s = reinterpret_cast<float *>(smem + L.xsum);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  int *meta = reinterpret_cast<int *>(smem + L.meta);
  uint32_t *emask = reinterpret_cast<uint32_t *>(meta);  // [32] expert presence bits
  int *wbase = meta + 32;                                 // [32] slots before word w
  int *slot_expert = meta + 64;                           // [256]
  int *slot_off = slot_expert + kDecMaxRows;              // [257]
  int *slot_rows = slot_off + kDecMaxRows + 1;            // [256] row ids grouped by slot
  int *ridx = slot_rows + kDecMaxRows;                    // [256] expert of row
  int *misc = ridx + kDecMaxRows;                         // [0] U, [1] abort, [2] epoch
  uint32_t *rmask = reinterpret_cast<uint32_t *>(misc + 8);  // [256 slots][8 words] rows of a slot
  float *rw = reinterpret_cast<float *>(rmask + kDecMaxRows * 8);  // [256] routing weights (fused)
  int *maxslot = reinterpret_cast<int *>(rw + kDecMaxRows);        // [16] highest slot of a token
  __shared__ int tok_lists[2][kDecMaxTok];
  __shared__ int ident[kDecMaxTok];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int team = warp / kTeamWarps, tw = warp % kTeamWarps, ttid = tid % kTeamThreads;
  const int bar_id = 1 + team;
  const int T = a.T, k = a.k, E = a.E, H = a.H, F = a.F;
  const int R = T * k, Gh = H / 64, Gf = F / 64, nt = dec_ntok_cols(T);
  const uint32_t stripA = (uint32_t)Gh * kBlkBytes, stripB = (uint32_t)Gf * kBlkBytes;
  const int G = gridDim.x;

  uint64_t *rbars = reinterpret_cast<uint64_t *>(smem + L.rbars);
  if (tid == 0) {
    for (int s = 0; s < a.nstages; ++s) mbar_init(&bars[s], 1);
    for (int w = 0; w < kDecWarps; ++w) mbar_init(&rbars[w], 1);
    fence_mbar_init();
  }
  if (tid < kDecMaxTok) ident[tid] = tid;
  if (kFp4 && tid < T) reinterpret_cast<unsigned int *>(xsum_s)[T + tid] = 0u;  // x row maxima
  if (tid < 32) emask[tid] = 0u;
  for (int i = tid; i < kDecMaxRows * 8; i += kDecThreads) rmask[i] = 0u;
  pdl_wait();  // inputs of this call may come from the previous kernel
  // The loads this setup needs go out together: x straight into shared
  // memory (int4; asynchronous), the call counter, the router logits.
  if (!kFp4) {
    for (int v = tid; v < T * H / 8; v += kDecThreads) cp_async_16(x_s + 8 * v, a.x + 8 * v);
    cp_async_commit();
  }
  const unsigned int ctrl0 = tid == kDecThreads - 1 ? a.ctrl[0] : 0u;
  __syncthreads();  // barrier initialisation and table clears are visible

  auto item_of = [&](int item, int nA, bool *isA, int *slot, int *sub) {
    if (item < nA) {
      *isA = true;
      *slot = item / (F / 16);
      *sub = item % (F / 16);
    } else {
      *isA = false;
      *slot = (item - nA) / (H / kDecOutRows);
      *sub = (item - nA) % (H / kDecOutRows);
    }
  };
  auto issue = [&](int item, int nA, int stage, uint64_t pol) {
    bool isA;
    int slot, sub;
    item_of(item, nA, &isA, &slot, &sub);
    const int e = slot_expert[slot];
    const uint8_t *src = isA ? a.gu + (size_t)e * a.gu_stride + (size_t)(2 * sub) * stripA
                             : a.dn + (size_t)e * a.dn_stride + (size_t)(4 * sub) * stripB;
    const uint32_t bytes = isA ? 2 * stripA : 4 * stripB;
    mbar_arrive_expect_tx(&bars[stage], bytes);
    bulk_g2s_evict_first(smem + L.stages + (size_t)stage * a.stage_bytes, src, bytes, &bars[stage],
                         pol);
  };

  // ---- router linear (with wr): each CTA computes the logits of its
  // experts e = blockIdx.x + G * (warp + kDecWarps * i), one warp per expert
  // row: lane l sums channels 8 l .. 8 l + 7 of every 256, in channel order,
  // in fp32 FMAs, the lanes' sums meet in an xor-shuffle tree (a fixed
  // order), and lane t
  // publishes token t's logit as a word {logit, epoch} for every CTA's
  // routing below.  All CTAs are resident together (cooperative launch) and
  // this phase waits on nothing but x, so every word gets written.
  if (kFused && !kFp4 && a.wr != nullptr) {
    const int Er = E - a.shared;
    if (tid == kDecThreads - 1) {
      const unsigned int ep = ctrl0 + 1u;  // this call's epoch; never 0 (zeroed words never match)
      misc[2] = (int)(ep == 0u ? 1u : ep);
    }
    // a warp's row comes into shared memory by one bulk copy (the stage
    // buffers are idle until the first weight copy, and 16 warps x 2 H bytes
    // fit in two stages); the first row's copy starts before waiting for x
    const int e_first = (int)blockIdx.x + G * warp;
    uint8_t *rowbuf = smem + L.stages + (size_t)warp * H * 2;
    auto fetch_row = [&](int e) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&rbars[warp], (uint32_t)H * 2u);
        bulk_g2s(rowbuf, a.wr + (size_t)e * H, (uint32_t)H * 2u, &rbars[warp]);
      }
    };
    if (e_first < Er) fetch_row(e_first);
    cp_async_wait_all();
    __syncthreads();
    const unsigned int ep = (unsigned int)misc[2];
    uint32_t rpar = 0;
    for (int e = e_first; e < Er; e += G * kDecWarps) {
      if (e != e_first) {
        __syncwarp();  // every lane is done with the previous row
        fence_proxy_async_smem();
        fetch_row(e);
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&rbars[warp], rpar, 1u << 22))) {
        if (lane == 0) atomicExch(a.err, DEVERR_DECODE_ROUTER_WAIT);
        break;  // the row never came: its words stay unwritten, and the routing's bounded waits give up
      }
      rpar ^= 1u;
      // tokens in groups of four (a loop over groups keeps the code short:
      // tokens past T cost issue slots even when predicated off)
      for (int t0 = 0; t0 < T; t0 += 4) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int c = 8 * lane; c < H; c += 256) {
          float wf[8];
          bf16x8_f32(*reinterpret_cast<const uint4 *>(rowbuf + (size_t)c * 2), wf);
#pragma unroll
          for (int tt = 0; tt < 4; ++tt) {
            if (t0 + tt < T) {
              float xf[8];
              bf16x8_f32(*reinterpret_cast<const uint4 *>(x_s + (size_t)(t0 + tt) * H + c), xf);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[tt] = __fmaf_rn(xf[i], wf[i], acc[tt]);
            }
          }
        }
        float mine = 0.f;
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          if (t0 + tt < T) {
            float v = acc[tt];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == tt) mine = v;
          }
        }
        if (lane < 4 && t0 + lane < T) {
          const int t = t0 + lane;
          a.lbuf[(size_t)t * Er + e] = ((unsigned long long)__float_as_uint(mine) << 32) | ep;
          if (a.logits_out) a.logits_out[(size_t)t * Er + e] = mine;
          // every CTA polls these words: push them out now (without the
          // fence they reached the pollers microseconds later; the h and row
          // words below measured slower with one)
          __threadfence();
        }
      }
    }
    // the rows were read by the generic proxy; the stages' next writers are
    // the weight copies (async proxy)
    fence_proxy_async_smem();
  }

  // ---- routing table.  Unique experts in increasing id ("slots"); the
  // first weight copies go out as soon as the slots are known.
  if (kFused) {  // warp t routes token t
    if (warp < T) {
      // with a shared expert the router scores the Er = E - 1 routed experts
      // and row kr = k - 1 is the shared expert's, weight 1
      const int kr = k - a.shared, Er = E - a.shared;
      uint32_t key[PER];
      if (!kFp4 && a.wr != nullptr) {
        // this token's logit words, all requested at once, then each one
        // polled again until it carries this call's epoch (bounded)
        const unsigned int ep = (unsigned int)misc[2];
        const unsigned long long *lw = a.lbuf + (size_t)warp * Er;
        unsigned long long wv[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) wv[i] = lane + 32 * i < Er ? ld_relaxed_u64(lw + lane + 32 * i) : 0ull;
        // every round reloads all of the lane's words still from an earlier
        // call, together
        uint32_t spins = 0;
        while (true) {
          uint32_t pending = 0;
#pragma unroll
          for (int i = 0; i < PER; ++i)
            if (lane + 32 * i < Er && (unsigned int)(wv[i] & 0xFFFFFFFFull) != ep) pending |= 1u << i;
          if (!pending) break;
          if (++spins > (1u << 22)) {  // the logits are used as read; the error word tells the caller
            atomicExch(a.err, DEVERR_DECODE_ROUTER_WAIT);
            break;
          }
          __nanosleep(32);
#pragma unroll
          for (int i = 0; i < PER; ++i)
            if ((pending >> i) & 1u) wv[i] = ld_relaxed_u64(lw + lane + 32 * i);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i)
          key[i] = lane + 32 * i < Er ? route_key(__uint_as_float((unsigned int)(wv[i] >> 32))) : 0u;
      } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int e = lane + 32 * i;
          key[i] = e < Er ? route_key(a.logits[(size_t)warp * Er + e]) : 0u;
        }
      }
      int j_idx;
      float j_w;
      route_token_keys<PER>(key, kr, &j_idx, &j_w);
      if (lane == kr) {  // only reached with a shared expert (kr < k)
        j_idx = Er;
        j_w = 1.0f;
      }
      if (lane < k) {
        ridx[warp * k + lane] = j_idx;
        rw[warp * k + lane] = j_w;
        atomicOr(&emask[j_idx >> 5], 1u << (j_idx & 31));
        if (blockIdx.x == 0 && a.idx_out && lane < kr) {
          a.idx_out[warp * kr + lane] = j_idx;
          a.w_out[warp * kr + lane] = j_w;
        }
      }
    }
  } else if (tid < R) {
    int e = a.idx[tid];
    e = (e < 0 || e >= E) ? 0 : e;  // out-of-range ids are outside the contract; stay memory safe
    ridx[tid] = e;
    atomicOr(&emask[e >> 5], 1u << (e & 31));
  }
  if (tid == kDecThreads - 1 && !(kFused && !kFp4 && a.wr != nullptr)) {  // (set above with wr)
    const unsigned int ep = ctrl0 + 1u;  // this call's epoch; never 0 (zeroed words never match)
    misc[2] = (int)(ep == 0u ? 1u : ep);
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t m = emask[lane];
    const int cnt = __popc(m);
    const int incl = warp_inclusive_scan(cnt);
    int base = incl - cnt;
    wbase[lane] = base;
    while (m) {
      slot_expert[base++] = 32 * lane + __ffs(m) - 1;
      m &= m - 1u;
    }
    const int U = __shfl_sync(0xffffffffu, incl, 31);
    __syncwarp();
    if (lane == 0) {
      misc[0] = U;
      misc[1] = 0;
    }
    // the CTA's first nstages items: lane q issues item q's copy into stage q
    // (the copies leave together instead of one after another)
    const int nA = U * (F / 16), nItems = nA + U * (H / kDecOutRows);
    const int myCount = (int)blockIdx.x < nItems ? (nItems - 1 - (int)blockIdx.x) / G + 1 : 0;
    if (lane < min(myCount, a.nstages)) issue(blockIdx.x + lane * G, nA, lane, policy_evict_first());
  }
  if (!kFp4) cp_async_wait_all();  // this thread's x copies
  __syncthreads();
  pdl_launch_dependents();
  // rows of each slot as a bit set; activation group sums
  int my_slot = 0;
  if (tid < R) {
    const int e = ridx[tid];
    my_slot = wbase[e >> 5] + __popc(emask[e >> 5] & ((1u << (e & 31)) - 1u));
    atomicOr(&rmask[my_slot * 8 + (tid >> 5)], 1u << (tid & 31));
  }
  if (!kFp4) {
    group_sums<true>(x_s, T, H, Gh, xsum_s, tid, kDecThreads);
  } else if (T * H / 2 <= 8 * kDecThreads) {  // all warps: channel pairs in registers
    float2 hv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int P = tid + kDecThreads * i;
      hv[i] = make_float2(0.f, 0.f);
      if (P < T * H / 2) {
        const uint32_t u = reinterpret_cast<const uint32_t *>(a.x)[P];  // channels 2P, 2P + 1 of x
        hv[i] = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
      }
    }
    nvfp4_pairs_f16<8>(hv, T, H, tid, kDecThreads, reinterpret_cast<unsigned int *>(xsum_s) + T, xsum_s, x_s,
                       [] { __syncthreads(); });
  } else if (warp < T) {  // warp t quantises token t: x_s = E2M1 * S_b (f16), xsum_s[t] = G
    const uint16_t *xr = a.x + (size_t)warp * H;
    const float G = nvfp4_row_f16(
        [&](int b, float (&v)[16]) {
          const uint4 *q = reinterpret_cast<const uint4 *>(xr + 16 * b);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint4 u4 = q[i];
            const uint32_t u[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              v[8 * i + 2 * jj] = __uint_as_float(u[jj] << 16);
              v[8 * i + 2 * jj + 1] = __uint_as_float(u[jj] & 0xFFFF0000u);
            }
          }
        },
        H / 16, x_s + (size_t)warp * H);
    if (lane == 0) xsum_s[warp] = G;
  }
  __syncthreads();
  const int U = misc[0];
  const unsigned int epoch = (unsigned int)misc[2];
  if (warp == 0) {  // slot sizes and their exclusive scan, 8 slots per lane
    int v[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sl = 8 * lane + i;
      int c = 0;
      if (sl < U)
#pragma unroll
        for (int w = 0; w < 8; ++w) c += __popc(rmask[sl * 8 + w]);
      v[i] = c;
      s += c;
    }
    int ex = warp_inclusive_scan(s) - s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sl = 8 * lane + i;
      if (sl < U) slot_off[sl] = ex;
      ex += v[i];
    }
    if (lane == 31) slot_off[U] = ex;
  }
  __syncthreads();
  if (tid < R) {  // rank of this row among its slot's rows, in row order
    int rank = __popc(rmask[my_slot * 8 + (tid >> 5)] & ((1u << (tid & 31)) - 1u));
    for (int w = 0; w < (tid >> 5); ++w) rank += __popc(rmask[my_slot * 8 + w]);
    slot_rows[slot_off[my_slot] + rank] = tid;
  }
  if (kFused && tid < T) {  // the slot whose down items combine token tid
    int mx = 0;
    for (int j = 0; j < k; ++j) {
      const int e = ridx[tid * k + j];
      mx = max(mx, wbase[e >> 5] + __popc(emask[e >> 5] & ((1u << (e & 31)) - 1u)));
    }
    maxslot[tid] = mx;
  }
  __syncthreads();

  const int nA = U * (F / 16), nItems = nA + U * (H / kDecOutRows);
  const int myCount = (int)blockIdx.x < nItems ? (nItems - 1 - (int)blockIdx.x) / G + 1 : 0;
  const uint64_t pol = policy_evict_first();
  int *tok_list = tok_lists[team];
  float *hsum_s = reinterpret_cast<float *>(smem + L.hsum) + (size_t)team * T * (kFp4 ? 2 : Gf);
  unsigned int *hrowmax = reinterpret_cast<unsigned int *>(hsum_s + T);  // NVFP4 only

  // ---- team `team` runs the CTA's items q = team, team + 2, ...
  bool aborted = false;
  int q_abort = 0;  // the item a team gave up on
  for (int q = team; q < myCount; q += 2) {
    const int item = blockIdx.x + q * G;
    const int stage = q % a.nstages;
    const uint32_t parity = (uint32_t)(q / a.nstages) & 1u;
    bool isA;
    int slot, sub;
    item_of(item, nA, &isA, &slot, &sub);
    const int r0 = slot_off[slot], ntok = slot_off[slot + 1] - r0;
    uint8_t *st = smem + L.stages + (size_t)stage * a.stage_bytes;
    if (ttid < kDecMaxTok) tok_list[ttid] = ttid < ntok ? slot_rows[r0 + ttid] / k : 0;
    uint16_t *h_s = reinterpret_cast<uint16_t *>(st + a.h_off);

    if (!isA) {
      // B item: poll this slot's h words until all carry this call's epoch
      // (bounded: only a broken contract waits for seconds), into the bf16
      // tile that sits behind the weights in this stage
      const int words = ntok * F;
      // NVFP4 with few enough values: channel pairs kept in registers for
      // the quantisation (no second pass over the words)
      const bool regs = kFp4 && words / 2 <= 8 * kTeamThreads;
      float2 hv[8];
      if (kFp4 && ttid < ntok) hrowmax[ttid] = 0u;
      uint32_t spins = 0;
      bool ready = false;
      while (true) {
        bool mine = true;
        if (regs) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int P = ttid + kTeamThreads * i;
            if (P < words / 2) {
              const int n = P / (F / 2), f = 2 * (P % (F / 2));
              const unsigned long long *wp = a.hbuf + (size_t)slot_rows[r0 + n] * F + f;
              const unsigned long long w0 = ld_relaxed_u64(wp), w1 = ld_relaxed_u64(wp + 1);
              if ((unsigned int)(w0 & 0xFFFFFFFFull) != epoch || (unsigned int)(w1 & 0xFFFFFFFFull) != epoch)
                mine = false;
              hv[i] = make_float2(__uint_as_float((uint32_t)(w0 >> 32)), __uint_as_float((uint32_t)(w1 >> 32)));
            }
          }
        } else
        for (int n = 0; n < ntok; ++n) {
          const unsigned long long *hr = a.hbuf + (size_t)slot_rows[r0 + n] * F;
          for (int f = ttid; f < F; f += kTeamThreads) {
            const unsigned long long w = ld_relaxed_u64(hr + f);
            if ((unsigned int)(w & 0xFFFFFFFFull) != epoch) mine = false;
            else if (!kFp4) h_s[(size_t)n * F + (f & ~63) + w4_kpos(f & 63)] = (uint16_t)(w >> 32);
          }
        }
        ready = !team_or(bar_id, !mine);
        if (ready || ++spins > a.h_polls) break;
        __nanosleep(100);
      }
      if (!ready) {
        if (ttid == 0) atomicExch(a.err, DEVERR_DECODE_H_WAIT);
        aborted = true;
        q_abort = q;
        break;
      }
      if (!kFp4) {
        group_sums(h_s, ntok, F, Gf, hsum_s, ttid, kTeamThreads);
      } else if (regs) {
        nvfp4_pairs_f16<8>(hv, ntok, F, ttid, kTeamThreads, hrowmax, hsum_s, h_s, [&] { team_sync(bar_id); });
        team_sync(bar_id);
      } else {  // warp per row: h (fp32) -> NVFP4 -> E2M1 * S_b in h_s, G in hsum_s
        for (int n = tw; n < ntok; n += kTeamWarps) {
          const unsigned long long *hr = a.hbuf + (size_t)slot_rows[r0 + n] * F;
          const float G = nvfp4_row_f16(
              [&](int b, float (&v)[16]) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  v[i] = __uint_as_float((uint32_t)(ld_relaxed_u64(hr + 16 * b + i) >> 32));
              },
              F / 16, h_s + (size_t)n * F);
          if (lane == 0) hsum_s[n] = G;
        }
        team_sync(bar_id);
      }
    }
    // wait for this item's weights (every thread observes the barrier)
    const bool landed = mbar_wait_bounded(&bars[stage], parity, 1u << 26);
    if (team_or(bar_id, !landed)) {  // only a copy stalled for seconds gets here
      if (ttid == 0) atomicExch(a.err, DEVERR_DECODE_H_WAIT);
      aborted = true;
      q_abort = q;
      break;
    }
    const int nbmax = ntok > 8 ? 2 : 1;
    float *red = reinterpret_cast<float *>(st);  // reused once the weights are consumed
    if (isA && a.starve_gate_up) {
      // test hook: the weights landed, but no h is computed or published
    } else if (isA) {
      float acc[2][2][4] = {};
      const uint8_t *base[2] = {st, st + stripA};
      if (kFp4) {
        if (nbmax == 2)
          fp4_warp_chunks<2, 2>(base, H, tw, kTeamWarps, x_s, H, tok_list, ntok, acc);
        else
          fp4_warp_chunks<1, 2>(base, H, tw, kTeamWarps, x_s, H, tok_list, ntok, acc);
      } else {
        const uint32_t wa[2] = {smem_u32(st), smem_u32(st) + stripA};
        const int ngw = tw < Gh ? (Gh - 1 - tw) / kTeamWarps + 1 : 0;
        if (nbmax == 2)
          w4_item<2, 2>(wa, tw, kTeamWarps, ngw, smem_u32(x_s), H, tok_list, ntok, smem_u32(xsum_s), Gh, acc);
        else
          w4_item<1, 2>(wa, tw, kTeamWarps, ngw, smem_u32(x_s), H, tok_list, ntok, smem_u32(xsum_s), Gh, acc);
      }
      team_sync(bar_id);  // all weights read
      frag_to_red(red + (size_t)(tw * 2 + 0) * 16 * nt, acc[0], nbmax, nt);
      frag_to_red(red + (size_t)(tw * 2 + 1) * 16 * nt, acc[1], nbmax, nt);
      team_sync(bar_id);
      // thread -> (row = ttid & 15, token n = ttid / 16): warp tw holds tokens
      // 2 tw and 2 tw + 1, so warps without tokens have nothing to do;
      // h = SiLU(g) * u
      const int row = ttid & 15, n = ttid >> 4;
      if (n < ntok) {
        float g = 0.f, u = 0.f;
#pragma unroll
        for (int w = 0; w < kTeamWarps; ++w) {
          g += red[(size_t)(w * 2 + 0) * 16 * nt + row * nt + n];
          u += red[(size_t)(w * 2 + 1) * 16 * nt + row * nt + n];
        }
        uint32_t hbits;
        if (kFp4) {  // the sums carry 2^-14; then the x and weight globals
          const float gs = __fmul_rn(xsum_s[tok_list[n]], a.g_gu[slot_expert[slot]]);
          g = __fmul_rn(__fmul_rn(g, 16384.0f), gs);
          u = __fmul_rn(__fmul_rn(u, 16384.0f), gs);
          hbits = __float_as_uint(g / (1.0f + expf(-g)) * u);
        } else {
          hbits = f32_to_bf16_bits(g / (1.0f + expf(-g)) * u);
        }
        const unsigned long long wv = ((unsigned long long)hbits << 32) | (unsigned long long)epoch;
        a.hbuf[(size_t)slot_rows[r0 + n] * F + 16 * sub + row] = wv;
      }
    } else {
      // warp -> strip (tw & 3), groups of parity (tw >> 2)
      float acc[1][2][4] = {};
      const uint8_t *base[1] = {st + (size_t)(tw & 3) * stripB};
      if (kFp4) {
        if (nbmax == 2)
          fp4_warp_chunks<2, 1>(base, F, tw >> 2, 2, h_s, F, ident, ntok, acc);
        else
          fp4_warp_chunks<1, 1>(base, F, tw >> 2, 2, h_s, F, ident, ntok, acc);
      } else {
        const uint32_t wa[1] = {smem_u32(st) + (uint32_t)(tw & 3) * stripB};
        const int g0 = tw >> 2, ngw = g0 < Gf ? (Gf - 1 - g0) / 2 + 1 : 0;
        if (nbmax == 2)
          w4_item<2, 1>(wa, g0, 2, ngw, smem_u32(h_s), F, ident, ntok, smem_u32(hsum_s), Gf, acc);
        else
          w4_item<1, 1>(wa, g0, 2, ngw, smem_u32(h_s), F, ident, ntok, smem_u32(hsum_s), Gf, acc);
      }
      team_sync(bar_id);  // all weights read
      frag_to_red(red + (size_t)tw * 16 * nt, acc[0], nbmax, nt);
      team_sync(bar_id);
      // thread -> (token n, output o of the 64): consecutive outputs, coalesced
      for (int v = ttid; v < kDecOutRows * ntok; v += kTeamThreads) {
        const int n = v >> 6, o = v & 63, strip = o >> 4, row = o & 15;
        float y = red[(size_t)strip * 16 * nt + row * nt + n] + red[(size_t)(strip + 4) * 16 * nt + row * nt + n];
        if (kFp4)
          y = __fmul_rn(__fmul_rn(y, 16384.0f), __fmul_rn(hsum_s[n], a.g_d[slot_expert[slot]]));
        const size_t oi = (size_t)slot_rows[r0 + n] * H + kDecOutRows * sub + o;
        if (kFused)
          a.ybuf[oi] = ((unsigned long long)__float_as_uint(y) << 32) | (unsigned long long)epoch;
        else
          a.y_rows[oi] = y;
      }
      if (kFused) {
        // combine the tokens of this slot whose highest slot is this one:
        // y[t][c] = sum over j (in order) of w[t][j] * row (t, j), polling the
        // rows of lower slots until they carry this call's epoch
        team_sync(bar_id);  // this item's own words are written
        bool ok = true;
        for (int v = ttid; v < ntok * kDecOutRows; v += kTeamThreads) {
          const int n = v / kDecOutRows, c = v % kDecOutRows;
          const int t = slot_rows[r0 + n] / k;
          if (maxslot[t] != slot) continue;
          float acc = 0.f;
          const unsigned long long *wp0 = a.ybuf + (size_t)t * k * H + kDecOutRows * sub + c;
          for (int j0 = 0; j0 < k && ok; j0 += 8) {
            // the (up to) eight rows' words are requested together, then
            // summed in j order; a word of an earlier call is polled again
            unsigned long long wv[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
              wv[jj] = j0 + jj < k ? ld_relaxed_u64(wp0 + (size_t)(j0 + jj) * H) : 0ull;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              if (j0 + jj >= k || !ok) break;
              uint32_t spins = 0;
              while ((unsigned int)(wv[jj] & 0xFFFFFFFFull) != epoch) {
                if (++spins > (1u << 22)) {
                  ok = false;
                  break;
                }
                __nanosleep(64);
                wv[jj] = ld_relaxed_u64(wp0 + (size_t)(j0 + jj) * H);
              }
              acc = __fadd_rn(acc, __fmul_rn(rw[t * k + j0 + jj], __uint_as_float((uint32_t)(wv[jj] >> 32))));
            }
          }
          a.y[(size_t)t * H + kDecOutRows * sub + c] = f32_to_bf16_bits(acc);
        }
        if (!ok) {
          atomicExch(a.err, DEVERR_DECODE_H_WAIT);
          aborted = true;
        }
      }
    }
    // generic-proxy writes to this stage are done; the next copy into it is
    // an async-proxy write
    fence_proxy_async_smem();
    if (team_or(bar_id, aborted)) {
      aborted = true;
      q_abort = q;
      break;
    }
    if (ttid == 0 && q + a.nstages < myCount) issue(blockIdx.x + (q + a.nstages) * G, nA, stage, pol);
  }

  // ---- aborted: let this team's in-flight copies land before leaving.  The
  // team has issued the copies of its items up to q_abort + nstages - 2 (the
  // first nstages at setup, then item q + nstages after finishing item q);
  // a stage's last issued copy is the one to wait for (phases complete in
  // order).
  if (aborted && ttid == 0) {
    const int hi = min(myCount - 1, q_abort + a.nstages - 2);
    for (int s = team; s < a.nstages && s <= hi; s += 2) {
      const int ql = s + (hi - s) / a.nstages * a.nstages;
      mbar_wait_bounded(&bars[s], (uint32_t)(ql / a.nstages) & 1u, 1u << 20);
    }
  }
  __syncthreads();
  // ---- last CTA out records this call's epoch for the next call
  if (tid == 0) {
    const unsigned int done = atomicAdd(&a.ctrl[1], 1u);
    if (done == (unsigned int)G - 1u) {
      a.ctrl[0] = epoch;
      a.ctrl[1] = 0u;
      __threadfence();
    }
  }
}

// One CTA per SM, as many weight stages as fit.  B items wait on A items of
// other CTAs, so every CTA must be resident at once: the launch is
// cooperative (the driver starts the grid only when all of its CTAs can run
// together, and refuses a grid that can never fit), and the grid is sized
// from the occupancy the kernel really gets.
template <int kFmt, bool kFused, int PER>
static moe_status decode_launch(DecodeArgs &a, bool pdl, cudaStream_t stream) {
  const int H = a.H, F = a.F, T = a.T, k = a.k;
  a.stage_bytes = dec_stage_bytes(T, H, F, &a.h_off);
  int dev = 0, sms = 0, smem_max = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const uint32_t cap = (uint32_t)smem_max - 1024;
  int nst = 8;  // even: the two teams own alternate stages
  while (nst > 2 && decode_smem_layout(kFmt, T, H, F, nst, a.stage_bytes).total > cap) nst -= 2;
  const DecodeSmem L = decode_smem_layout(kFmt, T, H, F, nst, a.stage_bytes);
  if (L.total > cap) return MOE_ERR_UNSUPPORTED_SHAPE;
  // the router rows (one per warp) are staged in the idle stage buffers
  if (a.wr && (size_t)nst * a.stage_bytes < (size_t)kDecWarps * 2u * (size_t)H) return MOE_ERR_UNSUPPORTED_SHAPE;
  a.nstages = nst;
  // per device: the shared-memory opt-in and the CTAs per SM it allows
  // (host threads may race here; both values are idempotent)
  static std::atomic<int> per_sm[64];
  if (dev < 0 || dev >= 64) {
    set_cuda_error(cudaErrorInvalidDevice);
    return MOE_ERR_CUDA;
  }
  if (per_sm[dev].load(std::memory_order_acquire) == 0) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<kFmt, kFused, PER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)cap);
    int occ = 0;
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<kFmt, kFused, PER>, kDecThreads, cap);
    if (e != cudaSuccess) {
      set_cuda_error(e);
      return MOE_ERR_CUDA;
    }
    if (occ < 1) return MOE_ERR_UNSUPPORTED_SHAPE;
    per_sm[dev].store(occ, std::memory_order_release);
  }
  const int maxItems = T * k * (F / 16 + H / kDecOutRows);
  const int grid = max(1, min(sms * per_sm[dev].load(std::memory_order_acquire), (maxItems + 1) / 2));

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<kFmt, kFused, PER>, a);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

static moe_status decode_check(const moe_w4_layer *layer, const uint16_t *x, const int32_t *idx,
                               int T, int k, const float *y_rows) {
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
  return MOE_OK;
}

static void decode_fill(DecodeArgs &a, const moe_w4_layer *layer, const uint16_t *x,
                        const int32_t *idx, int T, int k, float *y_rows, uint8_t *scratch) {
  a.logits = nullptr;
  a.y = nullptr;
  a.idx_out = nullptr;
  a.w_out = nullptr;
  a.ybuf = nullptr;
  a.gu = static_cast<const uint8_t *>(layer->gate_up);
  a.dn = static_cast<const uint8_t *>(layer->down);
  a.gu_stride = w4_packed_bytes(2 * layer->F, layer->H);
  a.dn_stride = w4_packed_bytes(layer->H, layer->F);
  a.x = x;
  a.idx = idx;
  a.y_rows = y_rows;
  a.g_gu = nullptr;
  a.g_d = nullptr;
  a.T = T;
  a.k = k;
  a.E = layer->E;
  a.H = layer->H;
  a.F = layer->F;
  a.ctrl = reinterpret_cast<unsigned int *>(scratch);
  a.hbuf = reinterpret_cast<unsigned long long *>(scratch + kDecCtrlBytes);
  a.h_polls = 1u << 20;
  a.starve_gate_up = 0;
  a.shared = 0;
  a.wr = nullptr;
  a.lbuf = nullptr;
  a.logits_out = nullptr;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_decode_workspace_bytes(int T, int k, int F) {
  if (T <= 0 || k <= 0 || F <= 0) return 0;
  return kDecCtrlBytes + sizeof(unsigned long long) * (size_t)T * k * F;
}

extern "C" MOE_API moe_status moe_ffn_w4a16_decode(const moe_w4_layer *layer, const uint16_t *x,
                                                   const int32_t *idx, int T, int k, float *y_rows,
                                                   void *ws, size_t ws_bytes,
                                                   moe_stream_t stream) {
  moe_status st = decode_check(layer, x, idx, T, k, y_rows);
  if (st != MOE_OK || T == 0) return st;
  if (!ws || ws_bytes < moe_decode_workspace_bytes(T, k, layer->F)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 16) return MOE_ERR_INVALID_ARG;
  DecodeArgs a;
  decode_fill(a, layer, x, idx, T, k, y_rows, static_cast<uint8_t *>(ws));
  a.err = device_error_word();
  if (!a.err) return MOE_ERR_CUDA;
  return decode_launch<kFmtW4, false, 8>(a, true, as_stream(stream));
}

extern "C" MOE_API moe_status moe_debug_starve_decode(const moe_w4_layer *layer, const uint16_t *x,
                                                      const int32_t *idx, int T, int k, float *y_rows,
                                                      void *ws, size_t ws_bytes, unsigned int polls,
                                                      moe_stream_t stream) {
  moe_status st = decode_check(layer, x, idx, T, k, y_rows);
  if (st != MOE_OK || T == 0) return st;
  if (!ws || ws_bytes < moe_decode_workspace_bytes(T, k, layer->F)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 16 || polls == 0) return MOE_ERR_INVALID_ARG;
  DecodeArgs a;
  decode_fill(a, layer, x, idx, T, k, y_rows, static_cast<uint8_t *>(ws));
  a.h_polls = polls;
  a.starve_gate_up = 1;
  a.err = device_error_word();
  if (!a.err) return MOE_ERR_CUDA;
  return decode_launch<kFmtW4, false, 8>(a, true, as_stream(stream));
}

extern "C" MOE_API size_t moe_decode_layer_workspace_bytes(int T, int k, int H, int F) {
  if (T <= 0 || k <= 0 || H <= 0 || F <= 0) return 0;
  return kDecCtrlBytes + sizeof(unsigned long long) * (size_t)T * k * ((size_t)F + (size_t)H);
}

// k: routed experts per token; shared: 1 = the layer's last expert is
// shared (every token's row k, weight 1), routing over the others.
// Exactly one of logits (given) and wr (router weights: the kernel computes
// the logits, optionally copied to logits_out) is non-null.
static moe_status decode_layer_w4(const moe_w4_layer *layer, const uint16_t *x, const float *logits,
                                  const uint16_t *wr, float *logits_out, int T, int k, int shared,
                                  uint16_t *y, int32_t *idx, float *w, void *ws, size_t ws_bytes,
                                  moe_stream_t stream) {
  if (!layer || T < 0 || k <= 0 || shared < 0 || shared > 1) return MOE_ERR_INVALID_ARG;
  const int E = layer->E, H = layer->H, F = layer->F, kk = k + shared;
  if (E <= shared || H <= 0 || F <= 0 || k > E - shared) return MOE_ERR_INVALID_ARG;
  if (H % 64 || F % 64 || E > kDecMaxE || T > kDecMaxTok || T * kk > kDecMaxRows || kk > 32)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!layer->gate_up || !layer->down || !x || (!logits == !wr) || !y) return MOE_ERR_INVALID_ARG;
  if ((idx == nullptr) != (w == nullptr)) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(layer->gate_up) % 16 ||
      reinterpret_cast<uintptr_t>(layer->down) % 16 || reinterpret_cast<uintptr_t>(x) % 16 ||
      reinterpret_cast<uintptr_t>(ws) % 16 || reinterpret_cast<uintptr_t>(wr) % 16)
    return MOE_ERR_INVALID_ARG;
  const size_t need = wr ? moe_decode_layer_router_workspace_bytes(T, k, shared, E, H, F)
                         : moe_decode_layer_workspace_bytes(T, kk, H, F);
  if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
  DecodeArgs a;
  decode_fill(a, layer, x, nullptr, T, kk, nullptr, static_cast<uint8_t *>(ws));
  a.shared = shared;
  a.logits = logits;
  a.wr = wr;
  a.logits_out = logits_out;
  a.lbuf = wr ? reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(ws) +
                                                      moe_decode_layer_workspace_bytes(T, kk, H, F))
              : nullptr;
  a.y = y;
  a.idx_out = idx;
  a.w_out = w;
  a.ybuf = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(ws) + kDecCtrlBytes +
                                                  sizeof(unsigned long long) * (size_t)T * kk * F);
  a.err = device_error_word();
  if (!a.err) return MOE_ERR_CUDA;
  if (E - shared <= 256) return decode_launch<kFmtW4, true, 8>(a, true, as_stream(stream));
  return decode_launch<kFmtW4, true, 32>(a, true, as_stream(stream));
}

extern "C" MOE_API moe_status moe_decode_layer_w4a16(const moe_w4_layer *layer, const uint16_t *x,
                                                     const float *logits, int T, int k,
                                                     uint16_t *y, int32_t *idx, float *w,
                                                     void *ws, size_t ws_bytes,
                                                     moe_stream_t stream) {
  if (!logits) return MOE_ERR_INVALID_ARG;
  return decode_layer_w4(layer, x, logits, nullptr, nullptr, T, k, 0, y, idx, w, ws, ws_bytes, stream);
}

extern "C" MOE_API moe_status moe_decode_layer_w4a16_shared(const moe_w4_layer *layer,
                                                            const uint16_t *x, const float *logits,
                                                            int T, int k, uint16_t *y, int32_t *idx,
                                                            float *w, void *ws, size_t ws_bytes,
                                                            moe_stream_t stream) {
  if (!logits) return MOE_ERR_INVALID_ARG;
  return decode_layer_w4(layer, x, logits, nullptr, nullptr, T, k, 1, y, idx, w, ws, ws_bytes, stream);
}

extern "C" MOE_API size_t moe_decode_layer_router_workspace_bytes(int T, int k, int shared, int E, int H,
                                                                  int F) {
  if (T <= 0 || k <= 0 || shared < 0 || shared > 1 || E <= shared || H <= 0 || F <= 0) return 0;
  return moe_decode_layer_workspace_bytes(T, k + shared, H, F) +
         sizeof(unsigned long long) * (size_t)T * (size_t)(E - shared);
}

extern "C" MOE_API moe_status moe_decode_layer_w4a16_router(const moe_w4_layer *layer, const uint16_t *x,
                                                            const uint16_t *wr, int T, int k, int shared,
                                                            uint16_t *y, int32_t *idx, float *w,
                                                            float *logits, void *ws, size_t ws_bytes,
                                                            moe_stream_t stream) {
  if (!wr) return MOE_ERR_INVALID_ARG;
  return decode_layer_w4(layer, x, nullptr, wr, logits, T, k, shared, y, idx, w, ws, ws_bytes, stream);
}

extern "C" MOE_API moe_status moe_decode_layer_nvfp4(const moe_nvfp4_layer *layer,
                                                     const uint16_t *x, const float *logits, int T,
                                                     int k, uint16_t *y, int32_t *idx, float *w,
                                                     void *ws, size_t ws_bytes,
                                                     moe_stream_t stream) {
  if (!layer || T < 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  const int E = layer->E, H = layer->H, F = layer->F;
  if (E <= 0 || H <= 0 || F <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (H % 256 || F % 256 || E > kDecMaxE || T > kDecMaxTok || T * k > kDecMaxRows || k > 32)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!layer->gate_up || !layer->down || !layer->g_gu || !layer->g_d || !x || !logits || !y)
    return MOE_ERR_INVALID_ARG;
  if ((idx == nullptr) != (w == nullptr)) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(layer->gate_up) % 16 ||
      reinterpret_cast<uintptr_t>(layer->down) % 16 || reinterpret_cast<uintptr_t>(x) % 16 ||
      reinterpret_cast<uintptr_t>(ws) % 16)
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_decode_layer_workspace_bytes(T, k, H, F)) return MOE_ERR_WORKSPACE;
  moe_w4_layer l4 = {E, H, F, layer->gate_up, layer->down};
  DecodeArgs a;
  decode_fill(a, &l4, x, nullptr, T, k, nullptr, static_cast<uint8_t *>(ws));
  a.gu_stride = (size_t)(2 * F / kBlkRows) * nvfp4_strip_bytes(H);
  a.dn_stride = (size_t)(H / kBlkRows) * nvfp4_strip_bytes(F);
  a.g_gu = layer->g_gu;
  a.g_d = layer->g_d;
  a.logits = logits;
  a.y = y;
  a.idx_out = idx;
  a.w_out = w;
  a.ybuf = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(ws) + kDecCtrlBytes +
                                                  sizeof(unsigned long long) * (size_t)T * k * F);
  a.err = device_error_word();
  if (!a.err) return MOE_ERR_CUDA;
  if (E <= 256) return decode_launch<kFmtNvfp4, true, 8>(a, true, as_stream(stream));
  return decode_launch<kFmtNvfp4, true, 32>(a, true, as_stream(stream));
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the decode call.
//
// Some callers cannot allocate device memory at all: plugins and embedded
// hosts whose device memory is owned and budgeted by the host application,
// and programs with a fixed memory plan that forbids any allocation once they
// have started serving.  They cannot supply the scratch workspace that
// moe_ffn_w4a16_decode needs, so this variant keeps its scratch (the call
// counter words and the h handoff buffer) in one fixed array in the library's
// own device memory instead.  The array is a module global: every GPU that
// loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
namespace moe {

constexpr size_t kStaticHBytes = 512 * 1024;  // T*k*F*8 bytes of h words at most
constexpr size_t kStaticScratchBytes = kDecCtrlBytes + kStaticHBytes;

static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device, looked up once per
// device (the lookup needs that device to be current).  Host threads may race
// on the first lookup; both find the same address.  A device reset
// (cudaDeviceReset) invalidates the cached address.
static uint8_t *static_scratch_address(moe_status *st) {
  static std::atomic<uint8_t *> addr[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    set_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
    *st = MOE_ERR_CUDA;
    return nullptr;
  }
  uint8_t *a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      set_cuda_error(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
      *st = MOE_ERR_CUDA;
      return nullptr;
    }
    a = static_cast<uint8_t *>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  *st = MOE_OK;
  return a;
}

}  // namespace moe

extern "C" MOE_API moe_status moe_ffn_w4a16_decode_static(const moe_w4_layer *layer,
                                                          const uint16_t *x, const int32_t *idx,
                                                          int T, int k, float *y_rows,
                                                          moe_stream_t stream) {
  moe_status st = decode_check(layer, x, idx, T, k, y_rows);
  if (st != MOE_OK) return st;
  // the fixed scratch holds at most kStaticHBytes / 8 h words
  if ((size_t)T * k * layer->F * sizeof(unsigned long long) > kStaticHBytes) return MOE_ERR_WORKSPACE;
  if (T == 0) return MOE_OK;
  uint8_t *scratch = static_scratch_address(&st);
  if (!scratch) return st;
  DecodeArgs a;
  decode_fill(a, layer, x, idx, T, k, y_rows, scratch);
  a.err = device_error_word();
  if (!a.err) return MOE_ERR_CUDA;
  // The array keeps whatever the previous call left in it.  The CTA counter
  // must start at zero, so clear it on the caller's stream before the launch;
  // the epoch word keeps counting up so that h words of earlier calls never
  // pass for this call's.
  cudaError_t e = cudaMemsetAsync(scratch + sizeof(unsigned int), 0, sizeof(unsigned int),
                                  as_stream(stream));
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return decode_launch<kFmtW4, false, 8>(a, false, as_stream(stream));
}
