// prefill.cu -- grouped expert FFN on the 5th-generation tensor cores.
//
// Prefill groups the rows of a batch by routed expert ("drama-rs", sections
// "Apple Silicon (MLX)" and "Layout": prefill runs a grouped MoE); every
// expert's rows then form a dense contraction with that expert's weights.
// Two launches of one kernel template.  A tile is a chunk of up to BN = 256
// rows of one expert and two 128-row weight blocks that share its activation
// tile (gate and up of 128 features, or 256 consecutive down outputs):
//   gate/up:  h = SiLU(D_gate) * D_up -> bf16 workspace [rows][F]
//   down:     -> y_perm bf16 [rows][H]
// A chunk of more than 128 rows puts the weights on the MMA's M (128 rows
// per block, one accumulator each) and the rows on N (trimmed to the valid
// rows).  A chunk of at most 128 rows is issued transposed: rows on M, the
// two contiguous weight blocks as one N = 256 operand, one MMA per k16 step.
// An MMA of M = 128, K = 16 costs about the same for any N up to ~200, so
// this halves the tensor time of few-row tiles.  Chunks of more than 128
// rows are scheduled first, in passes over the CTAs that alternate direction.
//
// Per 64-channel k block (one quantisation group):
//   int4 producer:   one TMA box per matrix of packed int4 blocks (8 strips)
//   act. producer:   TMA (128-byte swizzle) of the 64-row boxes holding rows
//   dequant warps:   int4 -> bf16, one FMA per code (q s + m in fp32, then
//                    nearest even) into the 128-byte-swizzled K-major smem
//                    layout the MMA reads
//   MMA thread:      tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in tensor
//                    memory), commit -> stages free
// then the dequant warps run the epilogue from tensor memory (tcgen05.ld):
// rows on N turn 32 outputs x 16 rows around in shared memory for 16-byte
// stores; rows on M write stretches of their own row.
// Every wait is bounded; a timeout raises the device error word.
#include <atomic>

#include "common.cuh"
#include "tcgen05.cuh"

namespace moe {

constexpr int kPfDqWarps = 16;   // warps 3..18: dequant, then epilogue
constexpr int kPfDqThreads = kPfDqWarps * 32;
constexpr int kPfThreads = (3 + kPfDqWarps) * 32;  // warp 0 int4 producer, 1 MMA, 2 activation producer
constexpr int kPfBM = 128;       // weight rows per matrix per tile
constexpr int kPfBN = 256;       // rows (tokens) per tile (the MMA's N is trimmed to the valid rows)
constexpr int kPfBK = 64;        // k block = one quantisation group
constexpr uint32_t kPfWaitPolls = 1u << 18;  // sleeping polls of up to 10 us: a bound of seconds

// Three rings: packed int4 blocks (deep: hides HBM latency, released by the
// dequant warps), bf16 weight tiles (dequant -> MMA), activation tiles (TMA ->
// MMA).
template <bool kGU>
struct PfCfg {
  // two 128-row MMA blocks per tile share each activation tile: gate and up
  // of 128 features, or 256 consecutive outputs of the down matrix (which
  // halves the down launch's re-reads of h)
  static constexpr int kMats = 2;
  static constexpr uint32_t kRawBytes = kMats * 8 * kBlkBytes;              // 8 strips per matrix
  static constexpr uint32_t kRawStride = (kRawBytes + 127) / 128 * 128;
  static constexpr uint32_t kABytes = kMats * kPfBM * kPfBK * 2;            // bf16 tiles
  static constexpr uint32_t kBBytes = kPfBN * kPfBK * 2;                    // activation tile
  static constexpr int kRawStages = 4;
  static constexpr int kAStages = 2;
  static constexpr int kBStages = 3;
  static constexpr uint32_t kTmemCols = kMats * kPfBN;  // 512: the two accumulators
  // layout: [A ring][B ring][raw ring][epilogue staging], 1024-aligned tiles
  static constexpr uint32_t kAOff = 0;
  static constexpr uint32_t kBOff = kAOff + kAStages * kABytes;
  static constexpr uint32_t kRawOff = kBOff + kBStages * kBBytes;
  static constexpr uint32_t kEpiOff = kRawOff + kRawStages * kRawStride;
  static constexpr uint32_t kEpiBytes = kPfDqWarps * 16 * 32 * 2;  // per warp: 16 rows x 32 outputs, bf16
  static constexpr uint32_t kTailOff = kEpiOff + kEpiBytes;
  // tail: barriers, TMEM address and flags, then two chunk tables of E + 1 ints (E <= 960)
  static constexpr uint32_t kSmemBytes = kTailOff + 1024 /*align slack*/ + 8192;
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct PrefillArgs {
  const uint8_t *w;        // expert weights (gate_up or down), expert e at e * w_stride
  size_t w_stride;
  const int32_t *offsets;  // [E + 1]
  uint16_t *out;           // gate/up: h [rows][F]; down: y_perm [rows][H]
  int *err;
  int E, K, rows;
  int n_sub;               // weight tiles per row chunk: F/128 (gate/up) or H/256 (down)
  int ld_out;              // F (gate/up) or H (down)
  int F;                   // gate/up: features per matrix (strip index of the up half)
  int spe;                 // strip pairs (gate/up) or strips (down) per expert
  uint32_t wait_polls;     // bound of every pipeline wait (sleeping polls)
  int starve_weights;      // test hook: the int4 producer issues no loads
};

// ---------------------------------------------------------------- tiles
// Row chunks of kPfBN rows, expert by expert.  A chunk of more than 128
// rows is "heavy" (two MMAs per k16 step), one of at most 128 rows "light"
// (one transposed MMA): an expert has n / 256 full chunks, plus a heavy or
// a light partial chunk.  Tiles are numbered heavy chunks first, then light
// ones, each chunk's n_sub weight tiles consecutive; heavy_start[e] /
// light_start[e] = first heavy / light chunk of expert e (exclusive scans).
struct TileInfo {
  int e, row0, nvalid, sub;
};
__device__ __forceinline__ TileInfo tile_info(int t, int n_sub, const int *heavy_start,
                                              const int *light_start, int E, const int32_t *offsets,
                                              int rows) {
  const int chunk = t / n_sub, nheavy = heavy_start[E];
  TileInfo ti;
  int o0, o1;
  if (chunk < nheavy) {
    ti.e = last_at_or_below(heavy_start, E, chunk);
    o0 = clamped_offset(offsets, ti.e, rows), o1 = clamped_offset(offsets, ti.e + 1, rows);
    ti.row0 = o0 + (chunk - heavy_start[ti.e]) * kPfBN;
  } else {
    ti.e = last_at_or_below(light_start, E, chunk - nheavy);
    o0 = clamped_offset(offsets, ti.e, rows), o1 = clamped_offset(offsets, ti.e + 1, rows);
    ti.row0 = o0 + (o1 - o0) / kPfBN * kPfBN;  // the partial chunk
  }
  ti.nvalid = min(kPfBN, o1 - ti.row0);
  ti.sub = t % n_sub;
  return ti;
}
template <bool kGU>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(PrefillArgs a, const __grid_constant__ CUtensorMap act_map,
                   const __grid_constant__ CUtensorMap w_map) {
  using C = PfCfg<kGU>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *tail = smem + C::kTailOff;  // barriers, tables
  uint64_t *raw_full = reinterpret_cast<uint64_t *>(tail);
  uint64_t *raw_empty = raw_full + C::kRawStages;
  uint64_t *a_full = raw_empty + C::kRawStages;
  uint64_t *a_empty = a_full + C::kAStages;
  uint64_t *b_full = a_empty + C::kAStages;
  uint64_t *b_empty = b_full + C::kBStages;
  uint64_t *tmem_full = b_empty + C::kBStages;
  uint64_t *tmem_empty = tmem_full + 1;
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(tmem_empty + 1);
  volatile int *abort_s = reinterpret_cast<volatile int *>(tmem_base_s + 1);
  int *ntiles_s = const_cast<int *>(abort_s) + 1;
  int *heavy_start = ntiles_s + 1;   // [E + 1]
  int *light_start = heavy_start + (a.E + 1);  // [E + 1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = a.K / kPfBK;

  if (tid == 0) {
    for (int s = 0; s < C::kRawStages; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kPfDqWarps);
    }
    for (int s = 0; s < C::kAStages; ++s) {
      mbar_init(&a_full[s], kPfDqWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < C::kBStages; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, kPfDqThreads);
    *abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_base_s, C::kTmemCols);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // chunk tables: exclusive scans of each expert's heavy and light chunks
  if (warp == 0) {
    int hcarry = 0, lcarry = 0;
    for (int e0 = 0; e0 < a.E; e0 += 32) {
      const int e = e0 + lane;
      const int n = e < a.E ? max(clamped_offset(a.offsets, e + 1, a.rows) - clamped_offset(a.offsets, e, a.rows), 0)
                            : 0;
      const int rem = n % kPfBN;
      const int hc = n / kPfBN + (rem > kPfBM ? 1 : 0), lc = (rem > 0 && rem <= kPfBM) ? 1 : 0;
      int hi = hc, li = lc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int hv = __shfl_up_sync(0xffffffffu, hi, o), lv = __shfl_up_sync(0xffffffffu, li, o);
        if (lane >= o) {
          hi += hv;
          li += lv;
        }
      }
      if (e < a.E) {
        heavy_start[e] = hcarry + hi - hc;
        light_start[e] = lcarry + li - lc;
      }
      hcarry += __shfl_sync(0xffffffffu, hi, 31);
      lcarry += __shfl_sync(0xffffffffu, li, 31);
    }
    if (lane == 0) {
      heavy_start[a.E] = hcarry;
      light_start[a.E] = lcarry;
      *ntiles_s = (hcarry + lcarry) * a.n_sub;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_s;
  const int ntiles = *ntiles_s;
  const int G = gridDim.x;
  auto fail = [&]() {
    atomicExch(a.err, DEVERR_PREFILL_WAIT);
    *abort_s = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ int4 producer
    if (lane == 0 && !a.starve_weights) {
      uint32_t it = 0;
      for (int i = 0, t = cta_tile(0, blockIdx.x, G); t < ntiles && !*abort_s; t = cta_tile(++i, blockIdx.x, G)) {
        const TileInfo ti = tile_info(t, a.n_sub, heavy_start, light_start, a.E, a.offsets, a.rows);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kRawStages;
          const uint32_t ph = (it / C::kRawStages) & 1u;
          if (!mbar_wait_sleep(&raw_empty[s], ph ^ 1u, a.wait_polls)) {
            fail();
            break;
          }
          uint8_t *raw = smem + C::kRawOff + s * C::kRawStride;
          mbar_arrive_expect_tx(&raw_full[s], C::kRawBytes);
          // one box per matrix: block kb of 8 strips.  gate/up: strip 2 r is
          // gate, 2 r + 1 up, of 16-feature block r (coordinates: strip pair,
          // gate/up); down: strips 16 sub + 8 m + i
          for (int m = 0; m < C::kMats; ++m) {
            if (kGU)
              tma_load_4d(raw + m * 8 * kBlkBytes, &w_map, 0, kb, m, ti.e * a.spe + ti.sub * 8, &raw_full[s]);
            else
              tma_load_3d(raw + m * 8 * kBlkBytes, &w_map, 0, kb, ti.e * a.spe + ti.sub * 16 + m * 8,
                          &raw_full[s]);
          }
        }
      }
      // aborted: the last load issued into each stage lands before the CTA
      // leaves (iterations [0, it) were issued)
      if (*abort_s)
        for (uint32_t j = it > (uint32_t)C::kRawStages ? it - C::kRawStages : 0u; j < it; ++j)
          mbar_wait_sleep(&raw_full[j % C::kRawStages], (j / C::kRawStages) & 1u, a.wait_polls);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int i = 0, t = cta_tile(0, blockIdx.x, G); t < ntiles && !*abort_s; t = cta_tile(++i, blockIdx.x, G)) {
        const TileInfo ti = tile_info(t, a.n_sub, heavy_start, light_start, a.E, a.offsets, a.rows);
        const int nbox = (ti.nvalid + 63) / 64;  // whole 64-row boxes covering the valid rows
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kBStages;
          const uint32_t ph = (it / C::kBStages) & 1u;
          if (!mbar_wait_sleep(&b_empty[s], ph ^ 1u, a.wait_polls)) {
            fail();
            break;
          }
          uint8_t *btile = smem + C::kBOff + s * C::kBBytes;
          mbar_arrive_expect_tx(&b_full[s], (uint32_t)nbox * 64u * 128u);
          for (int r = 0; r < nbox * 64; r += 64)
            tma_load_2d(btile + r * 128, &act_map, kb * kPfBK, ti.row0 + r, &b_full[s]);
        }
      }
      if (*abort_s)  // as for the int4 producer
        for (uint32_t j = it > (uint32_t)C::kBStages ? it - C::kBStages : 0u; j < it; ++j)
          mbar_wait_sleep(&b_full[j % C::kBStages], (j / C::kBStages) & 1u, a.wait_polls);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(smem + C::kAOff));
      const uint64_t bdesc0 = smem_desc_sw128(smem_u32(smem + C::kBOff));
      uint32_t it = 0, tcount = 0;
      for (int i = 0, t = cta_tile(0, blockIdx.x, G); t < ntiles && !*abort_s;
           t = cta_tile(++i, blockIdx.x, G), ++tcount) {
        const TileInfo ti = tile_info(t, a.n_sub, heavy_start, light_start, a.E, a.offsets, a.rows);
        // A tile of at most 128 rows is issued transposed (rows on M, the 256
        // weight rows on N): one MMA per k16 step instead of two.  An MMA
        // costs about as much at N = 16 as at N = 200, so this halves the
        // tensor time of the many few-row tiles.
        const bool swapped = ti.nvalid <= kPfBM;
        const uint32_t idesc = idesc_bf16_f32(swapped ? C::kMats * kPfBM : (ti.nvalid + 15) & ~15);
        if (!mbar_wait_sleep(tmem_empty, (tcount & 1u) ^ 1u, a.wait_polls)) {
          fail();
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int sa = it % C::kAStages, sb = it % C::kBStages;
          const uint32_t pa = (it / C::kAStages) & 1u, pb = (it / C::kBStages) & 1u;
          if (!mbar_wait_sleep(&b_full[sb], pb, a.wait_polls) ||
              !mbar_wait_sleep(&a_full[sa], pa, a.wait_polls)) {
            fail();
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors: the start-address field counts 16-byte units, so an
          // offset inside shared memory is added to it directly
          const uint64_t at = adesc0 + ((uint32_t)sa * C::kABytes >> 4);
          const uint64_t bt = bdesc0 + ((uint32_t)sb * C::kBBytes >> 4);
          if (swapped) {
            // D [128 rows][256 weight rows] = X [128][16] . W [256][16]^T: the two
            // 128-row weight tiles are contiguous, one 256-row operand
#pragma unroll
            for (int kk = 0; kk < kPfBK / 16; ++kk)
              tc_mma_bf16(tmem_base, bt + (kk * 32 >> 4), at + (kk * 32 >> 4), idesc, (kb | kk) ? 1u : 0u);
          } else {
            // one accumulator at a time: alternating accumulators between
            // consecutive MMAs costs about 15 % of the tensor rate at N = 256
#pragma unroll
            for (int m = 0; m < C::kMats; ++m)
#pragma unroll
              for (int kk = 0; kk < kPfBK / 16; ++kk)
                tc_mma_bf16(tmem_base + m * kPfBN, at + ((m * (kPfBM * 128) + kk * 32) >> 4), bt + (kk * 32 >> 4),
                            idesc, (kb | kk) ? 1u : 0u);
          }
          tc_commit(&a_empty[sa]);  // both operand stages are free once these MMAs have read them
          tc_commit(&b_empty[sb]);
        }
        if (!ok) break;
        tc_commit(tmem_full);  // accumulators complete
      }
    }
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    const int dw = warp - 3;            // 0..15
    const int quarter = warp & 3;       // TMEM lanes this warp may read
    const int cgrp = dw >> 2;           // epilogue: column group of this warp
    const int gi = lane >> 2, t4 = lane & 3;
    // This warp converts 16-row block rbk of both matrices in every k block:
    // words 2 wh and 2 wh + 1 of every lane's 16-byte fragment.
    const int rbk = dw >> 1, wh = dw & 1;
    // Byte offset of this lane's bf16 pair (channels 16 j + 2 t4 + 8 hk, +1;
    // j = 2 wh + jj) of row rbk * 16 + gi inside a matrix tile: 8-row atoms of
    // 1024 bytes, 128-byte rows, 16-byte chunk (2 j + hk) xor gi.  Row
    // rbk * 16 + gi + 8 is the next atom (+ 1024).
    uint32_t soff[2][2];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
      for (int hk = 0; hk < 2; ++hk)
        soff[jj][hk] = (uint32_t)(rbk * 2048 + gi * 128 + ((((2 * (2 * wh + jj) + hk) ^ gi) << 4) | (t4 << 2)));
    const uint32_t smem_s = smem_u32(smem);
    const uint32_t code_off = (uint32_t)(rbk * kBlkBytes + 16 * lane + 8 * wh);
    const uint32_t scale_off = (uint32_t)(rbk * kBlkBytes + kBlkCodeBytes + 4 * gi);
    uint32_t it = 0, tcount = 0;
    for (int i = 0, t = cta_tile(0, blockIdx.x, G); t < ntiles; t = cta_tile(++i, blockIdx.x, G), ++tcount) {
      const TileInfo ti = tile_info(t, a.n_sub, heavy_start, light_start, a.E, a.offsets, a.rows);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int sr = it % C::kRawStages, sa = it % C::kAStages;
        const uint32_t pr = (it / C::kRawStages) & 1u, pa = (it / C::kAStages) & 1u;
        const bool landed = mbar_wait_sleep(&raw_full[sr], pr, a.wait_polls) &&
                            mbar_wait_sleep(&a_empty[sa], pa ^ 1u, a.wait_polls);
        if (!landed || *abort_s) {
          if (!landed) fail();
          ok = false;
          break;
        }
        const uint32_t raw_s = smem_s + C::kRawOff + (uint32_t)sr * C::kRawStride;
        const uint32_t at_s = smem_s + C::kAOff + (uint32_t)sa * C::kABytes;
#pragma unroll
        for (int m = 0; m < C::kMats; ++m) {
          const uint32_t blk_s = raw_s + (uint32_t)(m * 8 * kBlkBytes);
          const uint2 cw = lds_v2(blk_s + code_off);
          const uint32_t sm0 = lds_b32(blk_s + scale_off), sm1 = lds_b32(blk_s + scale_off + 32);
          // q * s + m in fp32 from one FMA per code.  A nibble at bit p of a
          // word, OR-ed into the exponent pattern (150 - p) << 23, is the fp32
          // value v = 2^K + q (K = 23 - p), and v * s + (m - 2^K s) = q s + m.
          // The codes are first brought to bit 8, 12 or 16 (K = 15, 11, 7), so
          // the constant m - 2^K s is exact unless m and 2^K s lie more than
          // 2^11 apart in magnitude, and otherwise off by at most 2^-24 2^K |s|
          // (<= 2^-9 |s|, far below the bf16 rounding that follows).
          float sc[2], mn[2], c8[2], c12[2], c16[2];
          sc[0] = f16_bits_to_f32((uint16_t)(sm0 & 0xFFFFu));
          sc[1] = f16_bits_to_f32((uint16_t)(sm1 & 0xFFFFu));
          mn[0] = f16_bits_to_f32((uint16_t)(sm0 >> 16));
          mn[1] = f16_bits_to_f32((uint16_t)(sm1 >> 16));
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            c8[r] = __fmaf_rn(-32768.0f, sc[r], mn[r]);
            c12[r] = __fmaf_rn(-2048.0f, sc[r], mn[r]);
            c16[r] = __fmaf_rn(-128.0f, sc[r], mn[r]);
          }
          const uint32_t tile_s = at_s + (uint32_t)(m * (kPfBM * 128));
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const uint32_t w = jj ? cw.y : cw.x;
            const uint32_t wl = w << 8;   // nibbles 0, 1 at bits 8, 12
            const uint32_t wr = w >> 12;  // nibbles 5, 6, 7 at bits 8, 12, 16
            // nibble i (channel k) and i + 4 (k + 1) of pair i: hr = i & 1, hk = i >> 1
            const float v[4][2] = {
                {__uint_as_float((wl & 0x00000F00u) | (142u << 23)), __uint_as_float((w & 0x000F0000u) | (134u << 23))},
                {__uint_as_float((wl & 0x0000F000u) | (138u << 23)), __uint_as_float((wr & 0x00000F00u) | (142u << 23))},
                {__uint_as_float((w & 0x00000F00u) | (142u << 23)), __uint_as_float((wr & 0x0000F000u) | (138u << 23))},
                {__uint_as_float((w & 0x0000F000u) | (138u << 23)), __uint_as_float((wr & 0x000F0000u) | (134u << 23))}};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int hr = i & 1, hk = i >> 1;
              const float clo = i == 0 || i == 2 ? c8[hr] : c12[hr];
              const float chi = i == 0 || i == 3 ? c16[hr] : (i == 1 ? c8[hr] : c12[hr]);
              sts_b32(tile_s + soff[jj][hk] + hr * 1024,
                      cvt_bf16x2(__fmaf_rn(v[i][0], sc[hr], clo), __fmaf_rn(v[i][1], sc[hr], chi)));
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&a_full[sa]);
          mbar_arrive(&raw_empty[sr]);
        }
      }
      if (!ok) break;
      // ---- epilogue: accumulators of this tile; the four warps of a lane
      // quarter split the columns
      if (!mbar_wait_sleep(tmem_full, tcount & 1u, a.wait_polls)) {
        fail();
        break;
      }
      tc_fence_after();
      const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16);
      if (ti.nvalid <= kPfBM) {
        // transposed accumulators: lane quarter q holds rows 32 q + lane, the
        // columns are the tile's 256 weight rows (gate then up, or 256
        // consecutive outputs); the four warps of a quarter split the
        // columns and every thread writes a stretch of its own row
        const int r = quarter * 32 + lane;
        const bool live = r < ti.nvalid;
        uint16_t *orow = a.out + (size_t)(ti.row0 + (live ? r : 0)) * a.ld_out + ti.sub * (kGU ? kPfBM : 2 * kPfBM);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c0 = kGU ? cgrp * 32 + 16 * h : cgrp * 64 + 32 * h;
          uint32_t v0[16], v1[16];
          tmem_ld16_async(trow + c0, v0);                     // gate (or outputs c0 ..)
          tmem_ld16_async(trow + (kGU ? kPfBM : 16) + c0, v1);  // up (or outputs c0 + 16 ..)
          tmem_ld_wait();
          tmem_regs_after_wait(v0);
          tmem_regs_after_wait(v1);
          uint32_t pk[kGU ? 8 : 16];
#pragma unroll
          for (int c = 0; c < (kGU ? 8 : 16); ++c) {
            if (kGU) {
              const float g0 = __uint_as_float(v0[2 * c]), g1 = __uint_as_float(v0[2 * c + 1]);
              const float u0 = __uint_as_float(v1[2 * c]), u1 = __uint_as_float(v1[2 * c + 1]);
              pk[c] = cvt_bf16x2(__fdividef(g0, 1.0f + __expf(-g0)) * u0, __fdividef(g1, 1.0f + __expf(-g1)) * u1);
            } else {
              const uint32_t *v = c < 8 ? v0 : v1;
              pk[c] = cvt_bf16x2(__uint_as_float(v[(2 * c) & 15]), __uint_as_float(v[(2 * c + 1) & 15]));
            }
          }
          if (live) {
#pragma unroll
            for (int q = 0; q < (kGU ? 2 : 4); ++q)
              *reinterpret_cast<uint4 *>(orow + c0 + 8 * q) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      } else {
        // each warp turns its 32 outputs x 16 rows around in shared memory and
        // writes them as 16-byte vectors (row c: 64 bytes from 4 lanes)
        uint16_t *stage = reinterpret_cast<uint16_t *>(smem + C::kEpiOff) + dw * 16 * 32;
        const int fbase = ti.sub * (kGU ? kPfBM : 2 * kPfBM) + quarter * 32;  // first output of this warp
        for (int c0 = cgrp * 16; c0 < kPfBN; c0 += 64) {
          if (c0 >= ti.nvalid) break;  // uniform across the warp
          uint32_t v0[16], v1[16];
          tmem_ld16_async(trow + c0, v0);
          tmem_ld16_async(trow + kPfBN + c0, v1);
          tmem_ld_wait();
          tmem_regs_after_wait(v0);
          tmem_regs_after_wait(v1);
#pragma unroll
          for (int blk = 0; blk < (kGU ? 1 : 2); ++blk) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              float y;
              if (kGU) {
                const float g = __uint_as_float(v0[c]), u = __uint_as_float(v1[c]);
                y = __fdividef(g, 1.0f + __expf(-g)) * u;  // 0 once exp(-g) overflows
              } else {
                y = __uint_as_float(blk ? v1[c] : v0[c]);
              }
              stage[c * 32 + lane] = f32_to_bf16_bits(y);
            }
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int q = lane + 32 * r, c = q >> 2, part = q & 3;
              if (c0 + c < ti.nvalid) {
                const uint4 v = *reinterpret_cast<const uint4 *>(stage + c * 32 + 8 * part);
                *reinterpret_cast<uint4 *>(a.out + (size_t)(ti.row0 + c0 + c) * a.ld_out + fbase +
                                           blk * kPfBM + 8 * part) = v;
              }
            }
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tmem_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
// bf16 [rows][cols] row-major, boxes of 64 columns x 64 rows, 128-byte swizzle.
static bool make_act_map(CUtensorMap *map, const void *base, int rows, int cols) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed int4 weights of all E experts as 32-bit words: one 576-byte block
// (144 words) x K/64 blocks per strip x strips.  gate/up: strips as
// {gate, up} x strip pairs, box = block kb of 8 gate (or up) strips; down:
// box = block kb of 8 consecutive strips.
static bool make_w4_map(CUtensorMap *map, const void *base, int E, int N, int K, bool gate_up) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t KB = (cuuint64_t)K / kGroup, strip = KB * kBlkBytes;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  if (gate_up) {
    cuuint64_t dims[4] = {kBlkBytes / 4, KB, 2, (cuuint64_t)E * (N / 32)};
    cuuint64_t strides[3] = {kBlkBytes, strip, 2 * strip};
    cuuint32_t box[4] = {kBlkBytes / 4, 1, 1, 8};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  cuuint64_t dims[3] = {kBlkBytes / 4, KB, (cuuint64_t)E * (N / 16)};
  cuuint64_t strides[2] = {kBlkBytes, strip};
  cuuint32_t box[3] = {kBlkBytes / 4, 1, 8};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kGU>
static moe_status prefill_launch(const PrefillArgs &a, const CUtensorMap &map, const CUtensorMap &wmap,
                                 cudaStream_t stream) {
  using C = PfCfg<kGU>;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_done[64];  // per device; the attribute call is idempotent
  if (dev < 0 || dev >= 64) {
    set_cuda_error(cudaErrorInvalidDevice);
    return MOE_ERR_CUDA;
  }
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<kGU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
    if (e != cudaSuccess) {
      set_cuda_error(e);
      return MOE_ERR_CUDA;
    }
    attr_done[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_kernel<kGU>, a, map, wmap);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_prefill_workspace_bytes(int rows, int F) {
  if (rows <= 0 || F <= 0) return 0;
  return (size_t)rows * F * 2;
}

extern "C" MOE_API moe_status moe_ffn_grouped_prefill(const moe_w4_layer *layer,
                                                      const uint16_t *x_perm,
                                                      const int32_t *offsets, int rows,
                                                      uint16_t *y_perm, void *ws, size_t ws_bytes,
                                                      moe_stream_t stream) {
  if (!layer || rows < 0) return MOE_ERR_INVALID_ARG;
  const int E = layer->E, H = layer->H, F = layer->F;
  if (E <= 0 || H <= 0 || F <= 0) return MOE_ERR_INVALID_ARG;
  if (H % (2 * kPfBM) || F % kPfBM || E > 960) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!layer->gate_up || !layer->down || !x_perm || !offsets || !y_perm) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_prefill_workspace_bytes(rows, F)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(x_perm) % 16 || reinterpret_cast<uintptr_t>(ws) % 16 ||
      reinterpret_cast<uintptr_t>(y_perm) % 16 || reinterpret_cast<uintptr_t>(layer->gate_up) % 16 ||
      reinterpret_cast<uintptr_t>(layer->down) % 16)
    return MOE_ERR_INVALID_ARG;
  int *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  uint16_t *h = static_cast<uint16_t *>(ws);
  CUtensorMap xmap, hmap, gumap, dnmap;
  if (!make_act_map(&xmap, x_perm, rows, H) || !make_act_map(&hmap, h, rows, F) ||
      !make_w4_map(&gumap, layer->gate_up, E, 2 * F, H, true) ||
      !make_w4_map(&dnmap, layer->down, E, H, F, false)) {
    set_cuda_error(cudaErrorInvalidValue);
    return MOE_ERR_CUDA;
  }
  cudaStream_t s = as_stream(stream);
  PrefillArgs gu;
  gu.w = static_cast<const uint8_t *>(layer->gate_up);
  gu.w_stride = w4_packed_bytes(2 * F, H);
  gu.offsets = offsets;
  gu.out = h;
  gu.err = err;
  gu.E = E;
  gu.K = H;
  gu.rows = rows;
  gu.n_sub = F / kPfBM;
  gu.ld_out = F;
  gu.F = F;
  gu.spe = F / 16;  // strip pairs per expert
  gu.wait_polls = kPfWaitPolls;
  gu.starve_weights = 0;
  moe_status st = prefill_launch<true>(gu, xmap, gumap, s);
  if (st != MOE_OK) return st;
  PrefillArgs dn = gu;
  dn.w = static_cast<const uint8_t *>(layer->down);
  dn.w_stride = w4_packed_bytes(H, F);
  dn.out = y_perm;
  dn.K = F;
  dn.n_sub = H / (2 * kPfBM);
  dn.ld_out = H;
  dn.spe = H / 16;  // strips per expert
  return prefill_launch<false>(dn, hmap, dnmap, s);
}

extern "C" MOE_API moe_status moe_debug_starve_prefill(const moe_w4_layer *layer, const uint16_t *x_perm,
                                                       const int32_t *offsets, int rows, void *ws,
                                                       size_t ws_bytes, unsigned int polls,
                                                       moe_stream_t stream) {
  if (!layer || rows <= 0 || polls == 0) return MOE_ERR_INVALID_ARG;
  const int E = layer->E, H = layer->H, F = layer->F;
  if (E <= 0 || H <= 0 || F <= 0) return MOE_ERR_INVALID_ARG;
  if (H % (2 * kPfBM) || F % kPfBM || E > 960) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!layer->gate_up || !x_perm || !offsets) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_prefill_workspace_bytes(rows, F)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(x_perm) % 16 || reinterpret_cast<uintptr_t>(ws) % 16 ||
      reinterpret_cast<uintptr_t>(layer->gate_up) % 16)
    return MOE_ERR_INVALID_ARG;
  int *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  CUtensorMap xmap, gumap;
  if (!make_act_map(&xmap, x_perm, rows, H) || !make_w4_map(&gumap, layer->gate_up, E, 2 * F, H, true)) {
    set_cuda_error(cudaErrorInvalidValue);
    return MOE_ERR_CUDA;
  }
  PrefillArgs gu;
  gu.w = static_cast<const uint8_t *>(layer->gate_up);
  gu.w_stride = w4_packed_bytes(2 * F, H);
  gu.offsets = offsets;
  gu.out = static_cast<uint16_t *>(ws);
  gu.err = err;
  gu.E = E;
  gu.K = H;
  gu.rows = rows;
  gu.n_sub = F / kPfBM;
  gu.ld_out = F;
  gu.F = F;
  gu.spe = F / 16;
  gu.wait_polls = polls;
  gu.starve_weights = 1;
  return prefill_launch<true>(gu, xmap, gumap, as_stream(stream));
}
