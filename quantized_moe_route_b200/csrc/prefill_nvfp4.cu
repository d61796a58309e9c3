// prefill_nvfp4.cu -- grouped NVFP4 expert FFN on the block-scaled tensor
// cores (tcgen05.mma kind::mxf4nvf4, 16-channel E4M3 block scales).
//
// Prefill groups the rows of a batch by routed expert ("drama-rs", sections
// "Apple Silicon (MLX)" and "Layout"); with NVFP4 experts ("Drama 3 - NVFP4
// routed experts", section "Quantization") both operands of every expert's
// contraction are E2M1 codes with one E4M3 scale per 16 input channels, which
// the sm_100 tensor cores consume as they are: no dequantisation anywhere.
//   gate/up:  D_gate, D_up [128 features][N <= 80 rows] = W [128][H] . X[N][H]^T,
//             epilogue g, u = D * G_x * G_w; h = SiLU(g) * u -> fp32 [rows][F]
//   (h is re-quantised per row to NVFP4 between the two launches)
//   down:     D [128 outputs][N <= 128 rows] = W_down [128][F] . h[N][F]^T,
//             epilogue y = D * G_h * G_w -> bf16 y_perm [rows][H]
// Per stage of 256 channels:
//   warp 0      TMA: weight code tiles (the packed rows are stored with the
//               128-byte swizzle already applied, so a plain box is a ready
//               operand), weight scales, and only the 32-row boxes of
//               activation codes (128-byte swizzle on the fly) and scales that
//               hold the tile's rows
//   warp 2      rearranges the stage's scales into the tensor-memory scale
//               layout (per 64 channels: 32 rows x {4 row groups x 4 scales})
//   warp 1      tcgen05.cp of the scales into tensor memory, then four
//               block-scaled MMAs per matrix (K = 64 each), commit -> stage free
//   warps 4..11 epilogue from tensor memory (tcgen05.ld), two warps per lane
//               quarter; both launches keep two accumulator sets (gate/up
//               tiles of 80 rows, down tiles of 128) so the epilogue of one
//               tile overlaps the next tile's MMAs
// Every wait is bounded; a timeout raises the device error word.
#include <atomic>

#include "common.cuh"
#include "nvfp4.cuh"
#include "tcgen05.cuh"

namespace moe {

constexpr int kNpBM = 128;   // weight rows per matrix per tile (MMA M)
constexpr int kNpKT = 256;   // channels per stage: 128 code bytes per row
constexpr int kNpBoxRows = 32;  // activation rows per TMA box (a tile loads the boxes it needs)
constexpr int kNpEpiWarps = 8;  // warps 4..11: two per tensor-memory lane quarter
constexpr int kNpThreads = (4 + kNpEpiWarps) * 32;
constexpr uint32_t kNpWaitPolls = 1u << 18;  // sleeping polls of up to 10 us: a bound of seconds

template <bool kGU>
struct NpCfg {
  static constexpr int kMats = kGU ? 2 : 1;
  // rows per tile; the MMA's N is trimmed to the valid rows.  Gate/up tiles
  // take 80 rows so that two accumulator sets fit in tensor memory beside
  // the per-stage scales (the epilogue of one tile overlaps the next tile's
  // MMAs) with few enough tiles that no CTA takes more than three at 512
  // tokens.
  static constexpr int kBN = kGU ? 80 : 128;
  static constexpr int kBRows = (kBN + 31) / 32 * 32;  // rows of the activation buffers: whole 32-row boxes
  static constexpr int kStages = kGU ? 3 : 5;
  static constexpr uint32_t kACodes = kNpBM * 128;  // 16 KB per matrix
  static constexpr uint32_t kBCodes = kBRows * 128;  // 12 or 16 KB
  static constexpr uint32_t kARaw = 8 * 256;        // 8 strips x (4 x 64 scale bytes)
  // [rows][16 scale bytes]; the rearrangement reads 128 rows, past the end
  // of a shorter buffer into the stage's own atom area (rows it never uses)
  static constexpr uint32_t kBRaw = kBRows * 16;
  static constexpr uint32_t kAtom = 512;            // 128 rows x 4 scales, tensor-memory order
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kMats * kACodes;
  static constexpr uint32_t kOffARaw = kOffB + kBCodes;
  static constexpr uint32_t kOffBRaw = kOffARaw + kMats * kARaw;
  static constexpr uint32_t kOffAAtom = kOffBRaw + kBRaw;
  static constexpr uint32_t kOffBAtom = kOffAAtom + kMats * 4 * kAtom;
  static constexpr uint32_t kStageBytes = (kOffBAtom + 4 * kAtom + 1023) / 1024 * 1024;
  static constexpr uint32_t kATxBytes = kMats * (kACodes + kARaw);
  static constexpr uint32_t kBoxTxBytes = kNpBoxRows * (128 + 16);
  static constexpr uint32_t kTailOff = kStages * kStageBytes;
  static constexpr uint32_t kSmemBytes = kTailOff + 1024 /*align slack*/ + 4096;
  // tensor memory: kAcc accumulator sets of [kMats][BN] columns (down keeps
  // two, so the epilogue of one tile overlaps the next tile's MMAs), then
  // per stage the scales: A (kMats x 4 blocks of 64 channels x 4 columns),
  // B (4 x 4 columns)
  static constexpr int kAcc = 2;
  static constexpr uint32_t kAccCols = kMats * kBN;
  static constexpr uint32_t kSfCols = (kMats + 1) * 16;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kAcc * kAccCols + kStages * kSfCols <= kTmemCols, "tensor memory");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct NpArgs {
  const int32_t *offsets;  // [E + 1]
  const float *act_G;      // [rows] per-row activation globals
  const float *w_G;        // [E] weight globals of this matrix
  float *h_out;            // gate/up: h fp32 [rows][F]
  uint16_t *y_out;         // down: y_perm bf16 [rows][H]
  int *err;
  int E, K, rows;
  int n_sub;               // weight tiles per row chunk: F/128 or H/128
  int ld_out;              // F or H
  int spe;                 // strips (down) or strip pairs (gate/up) per expert
};

// ---------------------------------------------------------------- PTX
// smem -> tensor memory copy of 32 rows x 128 bits, replicated into the four
// 32-lane sub-partitions (the layout the block-scaled MMA reads scales from)
__device__ __forceinline__ void tc_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
__device__ __forceinline__ void tc_mma_nvf4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// Descriptor of a plain (unswizzled) K-major run of 8-row x 16-byte core
// matrices, 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_plain(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 16;
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  return d;
}
// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B (K-major), UE4M3
// scales, fp32 D, M = 128, N = n, K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int n) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kNpBM >> 4) << 24);
}

struct NpTile {
  int e, row0, nvalid, sub;
};
__device__ __forceinline__ NpTile np_tile(int t, int n_sub, const int *chunk_start, int E,
                                          const int32_t *offsets, int rows, int bn) {
  const int chunk = t / n_sub;
  int lo = 0, hi = E - 1;  // last expert with chunk_start[e] <= chunk
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (chunk_start[mid] <= chunk) lo = mid;
    else hi = mid - 1;
  }
  NpTile ti;
  ti.e = lo;
  ti.row0 = clamped_offset(offsets, lo, rows) + (chunk - chunk_start[lo]) * bn;
  ti.nvalid = min(bn, clamped_offset(offsets, lo + 1, rows) - ti.row0);
  ti.sub = t % n_sub;
  return ti;
}

template <bool kGU>
__global__ void __launch_bounds__(kNpThreads, 1)
    prefill_nvfp4_kernel(NpArgs a, const __grid_constant__ CUtensorMap wmap,
                         const __grid_constant__ CUtensorMap wsmap,
                         const __grid_constant__ CUtensorMap bmap,
                         const __grid_constant__ CUtensorMap bsmap) {
  using C = NpCfg<kGU>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem =
      reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *tail = smem + C::kTailOff;
  uint64_t *full = reinterpret_cast<uint64_t *>(tail);
  uint64_t *sfready = full + C::kStages;
  uint64_t *empty = sfready + C::kStages;
  uint64_t *tmem_full = empty + C::kStages;   // [kAcc]
  uint64_t *tmem_empty = tmem_full + C::kAcc;  // [kAcc]
  uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(tmem_empty + C::kAcc);
  volatile int *abort_s = reinterpret_cast<volatile int *>(tmem_base_s + 1);
  int *ntiles_s = const_cast<int *>(abort_s) + 1;
  int *chunk_start = ntiles_s + 1;  // [E + 1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KT = a.K / kNpKT;

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sfready[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kAcc; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], kNpEpiWarps * 32);
    }
    *abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_base_s, C::kTmemCols);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (warp == 0) {  // chunk table: chunk_start[e] = sum over e' < e of ceil(rows(e') / BN)
    int carry = 0;
    for (int e0 = 0; e0 < a.E; e0 += 32) {
      const int e = e0 + lane;
      const int n = e < a.E ? max(clamped_offset(a.offsets, e + 1, a.rows) - clamped_offset(a.offsets, e, a.rows), 0)
                            : 0;
      const int c = (max(n, 0) + C::kBN - 1) / C::kBN;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < a.E) chunk_start[e] = carry + incl - c;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      chunk_start[a.E] = carry;
      *ntiles_s = carry * a.n_sub;
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
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort_s; t += G) {
        const NpTile ti = np_tile(t, a.n_sub, chunk_start, a.E, a.offsets, a.rows, C::kBN);
        const int strip0 = ti.e * a.spe + 8 * ti.sub;  // first strip (pair) of the weight tile
        for (int kt = 0; kt < KT; ++kt, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait_sleep(&empty[s], ph ^ 1u, kNpWaitPolls)) {
            fail();
            break;
          }
          uint8_t *st = smem + s * C::kStageBytes;
          const int nbox = (ti.nvalid + kNpBoxRows - 1) / kNpBoxRows;
          mbar_arrive_expect_tx(&full[s], C::kATxBytes + (uint32_t)nbox * C::kBoxTxBytes);
          for (int m = 0; m < C::kMats; ++m) {
            if (kGU) {
              tma_load_4d(st + C::kOffA + m * C::kACodes, &wmap, kt * 128, 0, m, strip0, &full[s]);
              tma_load_3d(st + C::kOffARaw + m * C::kARaw, &wsmap, kt * 256, m, strip0, &full[s]);
            } else {
              tma_load_3d(st + C::kOffA, &wmap, kt * 128, 0, strip0, &full[s]);
              tma_load_2d(st + C::kOffARaw, &wsmap, kt * 256, strip0, &full[s]);
            }
          }
          for (int b = 0; b < nbox; ++b) {
            tma_load_2d(st + C::kOffB + b * kNpBoxRows * 128, &bmap, kt * 128, ti.row0 + b * kNpBoxRows,
                        &full[s]);
            tma_load_2d(st + C::kOffBRaw + b * kNpBoxRows * 16, &bsmap, kt * 16, ti.row0 + b * kNpBoxRows,
                        &full[s]);
          }
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale rearrangement
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += G) {
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1u;
        if (!mbar_wait_sleep(&full[s], ph, kNpWaitPolls) || *abort_s) {
          if (lane == 0 && !*abort_s) fail();
          ok = false;
          break;
        }
        uint8_t *st = smem + s * C::kStageBytes;
        // weights: raw [8 strips][4 blocks of 64][16 rows][4] -> per block,
        // words 4 l .. 4 l + 3 = tile rows l, l + 32, l + 64, l + 96 (row R
        // is row R % 16 of strip R / 16)
        for (int m = 0; m < C::kMats; ++m) {
          const uint32_t *raw = reinterpret_cast<const uint32_t *>(st + C::kOffARaw + m * C::kARaw);
          uint4 *atom = reinterpret_cast<uint4 *>(st + C::kOffAAtom + m * 4 * C::kAtom);
          const int rbase = (lane >> 4) * 64 + (lane & 15);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            atom[c * 32 + lane] = make_uint4(raw[rbase + c * 16], raw[rbase + 128 + c * 16],
                                             raw[rbase + 256 + c * 16], raw[rbase + 384 + c * 16]);
        }
        // activations: raw [128 rows][4 blocks][4] -> per block, row n at
        // 16 (n % 32) + 4 (n / 32): lane l moves rows l, l+32, l+64, l+96
        {
          const uint4 *braw = reinterpret_cast<const uint4 *>(st + C::kOffBRaw);
          uint4 *batom = reinterpret_cast<uint4 *>(st + C::kOffBAtom);
          const uint4 v0 = braw[lane], v1 = braw[lane + 32], v2 = braw[lane + 64], v3 = braw[lane + 96];
          batom[0 * 32 + lane] = make_uint4(v0.x, v1.x, v2.x, v3.x);
          batom[1 * 32 + lane] = make_uint4(v0.y, v1.y, v2.y, v3.y);
          batom[2 * 32 + lane] = make_uint4(v0.z, v1.z, v2.z, v3.z);
          batom[3 * 32 + lane] = make_uint4(v0.w, v1.w, v2.w, v3.w);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfready[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // descriptors: the start-address field counts 16-byte units, so an
      // offset inside shared memory is added to it directly
      const uint64_t dsw0 = smem_desc_sw128(smem_u32(smem)), dpl0 = smem_desc_plain(smem_u32(smem));
      uint32_t it = 0, tcount = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort_s; t += G, ++tcount) {
        const NpTile ti = np_tile(t, a.n_sub, chunk_start, a.E, a.offsets, a.rows, C::kBN);
        const uint32_t idesc = idesc_nvf4((ti.nvalid + 15) & ~15);
        const int ab = tcount % C::kAcc;
        const uint32_t acc0 = tmem_base + ab * C::kAccCols;
        if (!mbar_wait_sleep(&tmem_empty[ab], ((tcount / C::kAcc) & 1u) ^ 1u, kNpWaitPolls)) {
          fail();
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait_sleep(&sfready[s], ph, kNpWaitPolls)) {
            fail();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t so = (uint32_t)s * C::kStageBytes;  // stage offset
          const uint64_t sw = dsw0 + (so >> 4), pl = dpl0 + (so >> 4);
          const uint32_t sf0 = tmem_base + C::kAcc * C::kAccCols + s * C::kSfCols;
#pragma unroll
          for (int m = 0; m < C::kMats; ++m)
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
              tc_cp_32x128b_x4(sf0 + m * 16 + kb * 4, pl + ((C::kOffAAtom + (m * 4 + kb) * C::kAtom) >> 4));
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            tc_cp_32x128b_x4(sf0 + C::kMats * 16 + kb * 4, pl + ((C::kOffBAtom + kb * C::kAtom) >> 4));
          // one accumulator's four MMAs, then the other's
#pragma unroll
          for (int m = 0; m < C::kMats; ++m)
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
              tc_mma_nvf4(acc0 + m * C::kBN, sw + ((C::kOffA + m * C::kACodes + kb * 32) >> 4),
                          sw + ((C::kOffB + kb * 32) >> 4), idesc, sf0 + m * 16 + kb * 4,
                          sf0 + C::kMats * 16 + kb * 4, (kt | kb) ? 1u : 0u);
          tc_commit(&empty[s]);  // stage (and its tensor-memory scales) free once these MMAs are done
        }
        if (!ok) break;
        tc_commit(&tmem_full[ab]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // tensor-memory lane quarter of this warp
    const int half = (warp - 4) >> 2;  // the two warps of a quarter take alternate 16-column chunks
    uint32_t tcount = 0;
    for (int t = blockIdx.x; t < ntiles; t += G, ++tcount) {
      const NpTile ti = np_tile(t, a.n_sub, chunk_start, a.E, a.offsets, a.rows, C::kBN);
      const int ab = tcount % C::kAcc;
      // the tile's activation globals times the expert's weight global,
      // loaded while the MMAs run: lane l holds rows l, l + 32, ...
      const float wG = a.w_G[ti.e];
      float gl[C::kBRows / 32];
#pragma unroll
      for (int i = 0; i < C::kBRows / 32; ++i) {
        const int r = 32 * i + lane;
        gl[i] = r < ti.nvalid ? __fmul_rn(a.act_G[ti.row0 + r], wG) : 0.f;
      }
      if (!mbar_wait_sleep(&tmem_full[ab], (tcount / C::kAcc) & 1u, kNpWaitPolls) || *abort_s) {
        if (lane == 0 && !*abort_s) fail();
        break;
      }
      tc_fence_after();
      const int wrow = ti.sub * kNpBM + q * 32 + lane;  // feature (gate/up) or output channel (down)
      const uint32_t trow = tmem_base + ab * C::kAccCols + ((uint32_t)(q * 32) << 16);
#pragma unroll
      for (int i = 0; i < C::kBRows / 32; ++i) {
        const int c0 = 32 * i + 16 * half;  // rows c0 .. c0 + 15
        if (c0 >= ti.nvalid) break;
        uint32_t v0[16], v1[16];
        tmem_ld16_async(trow + c0, v0);
        if (kGU) tmem_ld16_async(trow + C::kBN + c0, v1);
        tmem_ld_wait();
        tmem_regs_after_wait(v0);
        if (kGU) tmem_regs_after_wait(v1);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float gs = __shfl_sync(0xffffffffu, gl[i], 16 * half + c);
          if (c0 + c < ti.nvalid) {
            const int p = ti.row0 + c0 + c;
            if (kGU) {
              const float g = __fmul_rn(__uint_as_float(v0[c]), gs);
              const float u = __fmul_rn(__uint_as_float(v1[c]), gs);
              a.h_out[(size_t)p * a.ld_out + wrow] = __fdividef(g, 1.0f + __expf(-g)) * u;
            } else {
              a.y_out[(size_t)p * a.ld_out + wrow] =
                  f32_to_bf16_bits(__fmul_rn(__uint_as_float(v0[c]), gs));
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tmem_empty[ab]);
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
static bool encode(CUtensorMap *map, const void *base, int rank, const cuuint64_t *dims,
                   const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void *>(base), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weight maps of one packed matrix kind for all E experts: codes as boxes of
// 8 strips x 16 rows x 128 bytes, scales as 8 strips x 256 bytes.
static bool make_weight_maps(CUtensorMap *codes, CUtensorMap *scales, const void *w, int E, int N,
                             int K, bool gate_up) {
  const cuuint64_t sb = nvfp4_strip_bytes(K);
  const uint8_t *base = static_cast<const uint8_t *>(w);
  if (gate_up) {
    const cuuint64_t pairs = (cuuint64_t)E * (N / 32);
    cuuint64_t cd[4] = {(cuuint64_t)K / 2, 16, 2, pairs};
    cuuint64_t cs[3] = {(cuuint64_t)K / 2, sb, 2 * sb};
    cuuint32_t cb[4] = {128, 16, 1, 8};
    cuuint64_t sd[3] = {(cuuint64_t)K, 2, pairs};
    cuuint64_t ss[2] = {sb, 2 * sb};
    cuuint32_t sbx[3] = {256, 1, 8};
    return encode(codes, base, 4, cd, cs, cb, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           encode(scales, base + (size_t)8 * K, 3, sd, ss, sbx, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  const cuuint64_t strips = (cuuint64_t)E * (N / 16);
  cuuint64_t cd[3] = {(cuuint64_t)K / 2, 16, strips};
  cuuint64_t cs[2] = {(cuuint64_t)K / 2, sb};
  cuuint32_t cb[3] = {128, 16, 8};
  cuuint64_t sd[2] = {(cuuint64_t)K, strips};
  cuuint64_t ss[1] = {sb};
  cuuint32_t sbx[2] = {256, 8};
  return encode(codes, base, 3, cd, cs, cb, CU_TENSOR_MAP_SWIZZLE_NONE) &&
         encode(scales, base + (size_t)8 * K, 2, sd, ss, sbx, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Activation maps: codes [rows][K/2] as boxes of 32 rows x 128 bytes with
// the 128-byte swizzle; scales [rows][K/16] as 32 rows x 16 bytes.
static bool make_act_maps(CUtensorMap *codes, CUtensorMap *scales, const uint8_t *c,
                          const uint8_t *sf, int rows, int K) {
  cuuint64_t cd[2] = {(cuuint64_t)K / 2, (cuuint64_t)rows};
  cuuint64_t cs[1] = {(cuuint64_t)K / 2};
  cuuint32_t cb[2] = {128, kNpBoxRows};
  cuuint64_t sd[2] = {(cuuint64_t)K / 16, (cuuint64_t)rows};
  cuuint64_t ss[1] = {(cuuint64_t)K / 16};
  cuuint32_t sbx[2] = {16, kNpBoxRows};
  return encode(codes, c, 2, cd, cs, cb, CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode(scales, sf, 2, sd, ss, sbx, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <bool kGU>
static moe_status np_launch(const NpArgs &a, const CUtensorMap &wm, const CUtensorMap &wsm,
                            const CUtensorMap &bm, const CUtensorMap &bsm, cudaStream_t stream) {
  using C = NpCfg<kGU>;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_done[64];  // per device; the attribute call is idempotent
  if (dev < 0 || dev >= 64) {
    set_cuda_error(cudaErrorInvalidDevice);
    return MOE_ERR_CUDA;
  }
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(prefill_nvfp4_kernel<kGU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
    if (e != cudaSuccess) {
      set_cuda_error(e);
      return MOE_ERR_CUDA;
    }
    attr_done[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kNpThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_nvfp4_kernel<kGU>, a, wm, wsm, bm, bsm);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Workspace sections (each 256-byte aligned): h fp32 [rows][F], h codes
// [rows][F/2], h scales [rows][F/16], h globals [rows].
struct NpWs {
  size_t h, hc, hs, hg, total;
};
static NpWs np_ws(int rows, int F) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  NpWs w;
  w.h = 0;
  w.hc = up(w.h + (size_t)rows * F * 4);
  w.hs = up(w.hc + (size_t)rows * F / 2);
  w.hg = up(w.hs + (size_t)rows * F / 16);
  w.total = up(w.hg + (size_t)rows * 4);
  return w;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_prefill_nvfp4_workspace_bytes(int rows, int F) {
  if (rows <= 0 || F <= 0) return 0;
  return np_ws(rows, F).total;
}

extern "C" MOE_API moe_status moe_ffn_grouped_prefill_nvfp4(
    const moe_nvfp4_layer *layer, const uint8_t *x_codes, const uint8_t *x_sf, const float *x_G,
    const int32_t *offsets, int rows, uint16_t *y_perm, void *ws, size_t ws_bytes,
    moe_stream_t stream) {
  if (!layer || rows < 0) return MOE_ERR_INVALID_ARG;
  const int E = layer->E, H = layer->H, F = layer->F;
  if (E <= 0 || H <= 0 || F <= 0) return MOE_ERR_INVALID_ARG;
  if (H % kNpKT || F % kNpKT || E > 960) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!layer->gate_up || !layer->down || !layer->g_gu || !layer->g_d || !x_codes || !x_sf ||
      !x_G || !offsets || !y_perm)
    return MOE_ERR_INVALID_ARG;
  const NpWs w = np_ws(rows, F);
  if (!ws || ws_bytes < w.total) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(x_codes) % 16 || reinterpret_cast<uintptr_t>(x_sf) % 16 ||
      reinterpret_cast<uintptr_t>(ws) % 256 || reinterpret_cast<uintptr_t>(y_perm) % 16 ||
      reinterpret_cast<uintptr_t>(layer->gate_up) % 16 || reinterpret_cast<uintptr_t>(layer->down) % 16)
    return MOE_ERR_INVALID_ARG;
  int *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  float *h = reinterpret_cast<float *>(wsb + w.h);
  uint8_t *hc = wsb + w.hc, *hs = wsb + w.hs;
  float *hg = reinterpret_cast<float *>(wsb + w.hg);
  CUtensorMap guc, gus, dnc, dns, xc, xs, hcm, hsm;
  if (!make_weight_maps(&guc, &gus, layer->gate_up, E, 2 * F, H, true) ||
      !make_weight_maps(&dnc, &dns, layer->down, E, H, F, false) ||
      !make_act_maps(&xc, &xs, x_codes, x_sf, rows, H) || !make_act_maps(&hcm, &hsm, hc, hs, rows, F)) {
    set_cuda_error(cudaErrorInvalidValue);
    return MOE_ERR_CUDA;
  }
  cudaStream_t s = as_stream(stream);
  NpArgs gu;
  gu.offsets = offsets;
  gu.act_G = x_G;
  gu.w_G = layer->g_gu;
  gu.h_out = h;
  gu.y_out = nullptr;
  gu.err = err;
  gu.E = E;
  gu.K = H;
  gu.rows = rows;
  gu.n_sub = F / kNpBM;
  gu.ld_out = F;
  gu.spe = F / 16;
  moe_status st = np_launch<true>(gu, guc, gus, xc, xs, s);
  if (st != MOE_OK) return st;
  // h -> NVFP4, one global per row (the format's per-row quantiser)
  st = moe_quantize_nvfp4_rows(h, 1, rows, F, nullptr, 1, hc, hs, hg, stream);
  if (st != MOE_OK) return st;
  NpArgs dn = gu;
  dn.act_G = hg;
  dn.w_G = layer->g_d;
  dn.h_out = nullptr;
  dn.y_out = y_perm;
  dn.K = F;
  dn.n_sub = H / kNpBM;
  dn.ld_out = H;
  dn.spe = H / 16;
  return np_launch<false>(dn, dnc, dns, hcm, hsm, s);
}
