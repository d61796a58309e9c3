// decode_common.cuh -- pieces shared by the decode kernels: tensor-core
// fragments built from packed int4 / NVFP4 codes, the group-affine fold,
// activation group sums, in-kernel NVFP4 quantisation of activation rows,
// and team barriers.
//
// int4: a packed 32-bit word holds the eight 4-bit codes one lane needs for
// one m16n8k16 A fragment; OR-ing 0x4300 into each 16-bit half turns code q
// into the bf16 value 128 + q exactly.  The tensor core forms
// D = sum (128 + q) x in fp32 over one 64-channel group, and the group's
// affine map is applied once per output and token:
//   sum_k (q s + m) x_k = s D + (m - 128 s) X,   X = sum_k x_k.
// NVFP4 ("Drama 3 - NVFP4 routed experts", section "Quantization"): a code
// word gives two f16 fragment halves by moving the 3 magnitude bits to bits
// 9..11 and the sign to bit 15, which is the E2M1 value times 2^-14 for every
// code (0.5 lands on the f16 subnormal 2^-15); one m16n8k16 step is one
// 16-channel block, whose weight scale is applied to that step's result.
#pragma once
#include "common.cuh"
#include "nvfp4.cuh"

namespace moe {
constexpr int kDecWarps = 16;             // two teams of eight warps
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kTeamWarps = 8;
constexpr int kTeamThreads = kTeamWarps * 32;
constexpr int kDecMaxTok = 16;   // tokens per expert per call (two n8 blocks)
constexpr int kDecMaxRows = 256; // T * k
constexpr int kDecMaxE = 1024;
constexpr int kDecOutRows = 64;  // outputs per B item (4 strips)
constexpr size_t kDecCtrlBytes = 4096;  // workspace head: epoch, done counter
constexpr int kFmtW4 = 0, kFmtNvfp4 = 1;

// token columns of the tensor-core tiles: one n8 block, or two above 8 tokens
__host__ __device__ inline int dec_ntok_cols(int T) { return T > 8 ? 16 : 8; }

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Barriers of one team (named barrier 1 + team, 256 threads).
__device__ __forceinline__ void team_sync(int id) {
  asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool team_or(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// eight bf16 (16 bytes) -> fp32, exact
__device__ __forceinline__ void bf16x8_f32(const uint4 &v, float f[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// (a & m) | c as one three-input logic instruction (written out: the
// compiler otherwise splits the mask and the OR into two)
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "r"(c));
  return d;
}

// The 4 A-fragment registers of one k16 step from one packed word: each
// 16-bit half becomes the bf16 value 128 + q.
__device__ __forceinline__ void w4_frag(uint32_t w, uint32_t a[4]) {
  const uint32_t M = 0x000F000Fu, C = 0x43004300u;
  a[0] = and_or(w, M, C);
  a[1] = and_or(w >> 4, M, C);
  a[2] = and_or(w >> 8, M, C);
  a[3] = and_or(w >> 12, M, C);
}

struct GroupAffine {
  float s0, c0, s1, c1;  // rows g and g+8: scale and (min - 128 scale)
};
__device__ __forceinline__ GroupAffine load_affine(const uint8_t *blk, int gi) {
  const uint32_t lo = *reinterpret_cast<const uint32_t *>(blk + kBlkCodeBytes + 4 * gi);
  const uint32_t hi = *reinterpret_cast<const uint32_t *>(blk + kBlkCodeBytes + 4 * (gi + 8));
  GroupAffine A;
  A.s0 = f16_bits_to_f32((uint16_t)(lo & 0xFFFFu));
  A.s1 = f16_bits_to_f32((uint16_t)(hi & 0xFFFFu));
  A.c0 = __fmaf_rn(-128.f, A.s0, f16_bits_to_f32((uint16_t)(lo >> 16)));
  A.c1 = __fmaf_rn(-128.f, A.s1, f16_bits_to_f32((uint16_t)(hi >> 16)));
  return A;
}

// acc += s * D + (m - 128 s) * X for this lane's four D-fragment entries.
__device__ __forceinline__ void fold(float acc[4], const float d[4], const float xs[4],
                                     const GroupAffine &A) {
  acc[0] = __fmaf_rn(A.c0, xs[0], __fmaf_rn(A.s0, d[0], acc[0]));
  acc[1] = __fmaf_rn(A.c0, xs[1], __fmaf_rn(A.s0, d[1], acc[1]));
  acc[2] = __fmaf_rn(A.c1, xs[2], __fmaf_rn(A.s1, d[2], acc[2]));
  acc[3] = __fmaf_rn(A.c1, xs[3], __fmaf_rn(A.s1, d[3], acc[3]));
}

// Shared-memory order of the 64 activations of a group (int4 path): channel
// k = 16 j + 8 hi + 2 t + lo sits at 16 t + 4 j + 2 hi + lo, so lane t's B
// fragments of the group's four k16 steps are 16 consecutive values (two
// 16-byte loads).
__host__ __device__ constexpr int w4_kpos(int k) {
  return 16 * ((k & 7) >> 1) + 4 * (k >> 4) + 2 * ((k >> 3) & 1) + (k & 1);
}

// One warp: NG 64-channel groups and NMAT matrices (gate and up, or down) of
// 16 rows each, against up to 16 activation rows held in shared memory as
// bf16 [n][ld] in w4_kpos order, whose per-group sums are gsum[n][g].  The A
// fragments of a group are built once and reused for both token blocks.
// Columns n >= ntok read row tok_of[0]; their results are never used.
template <int NB, int NMAT, int NG>
__device__ __forceinline__ void group_mma(const uint8_t *const (&blk)[NG][NMAT],
                                          const uint16_t *act, int ld, const int (&gidx)[NG],
                                          const int *tok_of, int ntok, const float *gsum,
                                          int gsum_ld, float acc[NMAT][2][4]) {
  const int lane = threadIdx.x & 31, gi = lane >> 2, t4 = lane & 3;
  uint32_t af[NG][NMAT][4][4];
  GroupAffine aff[NG][NMAT];
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      const uint4 cw = *reinterpret_cast<const uint4 *>(blk[g][m] + 16 * lane);
      w4_frag(cw.x, af[g][m][0]);
      w4_frag(cw.y, af[g][m][1]);
      w4_frag(cw.z, af[g][m][2]);
      w4_frag(cw.w, af[g][m][3]);
      aff[g][m] = load_affine(blk[g][m], gi);
    }
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int n = nb * 8 + gi;  // this lane's B column (token slot)
    const uint16_t *arow = act + (size_t)tok_of[n < ntok ? n : 0] * ld + 16 * t4;
    const int na = nb * 8 + 2 * t4, nb1 = na + 1;  // this lane's D columns
    const float *ga = gsum + (size_t)tok_of[na < ntok ? na : 0] * gsum_ld;
    const float *gb = gsum + (size_t)tok_of[nb1 < ntok ? nb1 : 0] * gsum_ld;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const uint4 q0 = *reinterpret_cast<const uint4 *>(arow + 64 * gidx[g]);
      const uint4 q1 = *reinterpret_cast<const uint4 *>(arow + 64 * gidx[g] + 8);
      const uint32_t b[4][2] = {{q0.x, q0.y}, {q0.z, q0.w}, {q1.x, q1.y}, {q1.z, q1.w}};
      const float xa = ga[gidx[g]], xb = gb[gidx[g]];
      const float xs[4] = {xa, xb, xa, xb};
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_bf16_16816(d, af[g][m][j], b[j][0], b[j][1]);
        fold(acc[m][nb], d, xs, aff[g][m]);
      }
    }
  }
}

// group_mma over a warp's groups first, first + step, ... < ngroups: two
// groups at a time for one token block, one at a time for two.
template <int NB, int NMAT>
__device__ __forceinline__ void warp_groups(const uint8_t *const (&mat_base)[NMAT], int first,
                                            int step, int ngroups, const uint16_t *act, int ld,
                                            const int *tok_of, int ntok, const float *gsum,
                                            int gsum_ld, float acc[NMAT][2][4]) {
  int g = first;
  if (NB == 1) {
    for (; g + step < ngroups; g += 2 * step) {
      const uint8_t *blk[2][NMAT];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        blk[0][m] = mat_base[m] + (size_t)g * kBlkBytes;
        blk[1][m] = mat_base[m] + (size_t)(g + step) * kBlkBytes;
      }
      const int gidx[2] = {g, g + step};
      group_mma<NB, NMAT, 2>(blk, act, ld, gidx, tok_of, ntok, gsum, gsum_ld, acc);
    }
  }
  for (; g < ngroups; g += step) {
    const uint8_t *blk[1][NMAT];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) blk[0][m] = mat_base[m] + (size_t)g * kBlkBytes;
    const int gidx[1] = {g};
    group_mma<NB, NMAT, 1>(blk, act, ld, gidx, tok_of, ntok, gsum, gsum_ld, acc);
  }
}

// A warp's D-fragment accumulators -> red[row][token] (nt token columns).
__device__ __forceinline__ void frag_to_red(float *red, const float acc[2][4], int nbmax, int nt) {
  const int lane = threadIdx.x & 31, gi = lane >> 2, t4 = lane & 3;
  for (int nb = 0; nb < nbmax; ++nb) {
    const int n = nb * 8 + 2 * t4;
    red[gi * nt + n] = acc[nb][0];
    red[gi * nt + n + 1] = acc[nb][1];
    red[(gi + 8) * nt + n] = acc[nb][2];
    red[(gi + 8) * nt + n + 1] = acc[nb][3];
  }
}

// Sums of 64 consecutive bf16 values: rows [nrows][ld] -> out[n][g] for the
// first ngroups groups; eight threads per sum, one 16-byte vector each.
// `t` / `nthreads`: this thread's index among the participating threads
// (a multiple of 32).  With kReorder, the group is also rewritten in place in
// w4_kpos order (the eight threads of a group share a warp).
template <bool kReorder = false>
__device__ __forceinline__ void group_sums(uint16_t *rows, int nrows, int ld, int ngroups,
                                           float *out, int t, int nthreads) {
  const int tasks = nrows * ngroups * 8;
  for (int v = t; v < ((tasks + nthreads - 1) / nthreads) * nthreads; v += nthreads) {
    float s = 0.f;
    const int task = v >> 3, part = v & 7;
    uint16_t *grp = rows;
    uint32_t u[4] = {0u, 0u, 0u, 0u};
    if (v < tasks) {
      const int n = task / ngroups, g = task % ngroups;
      grp = rows + (size_t)n * ld + 64 * g;
      const uint4 q = *reinterpret_cast<const uint4 *>(grp + 8 * part);
      u[0] = q.x, u[1] = q.y, u[2] = q.z, u[3] = q.w;
#pragma unroll
      for (int i = 0; i < 4; ++i) s += __uint_as_float(u[i] << 16) + __uint_as_float(u[i] & 0xFFFF0000u);
    }
    if (kReorder) {
      __syncwarp();  // the whole group is in registers before any of it moves
      if (v < tasks)
#pragma unroll
        for (int i = 0; i < 4; ++i)  // channels 8 part + 2 i, + 1
          *reinterpret_cast<uint32_t *>(grp + w4_kpos(8 * part + 2 * i)) = u[i];
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (v < tasks && part == 0) out[task] = s;
  }
}

// ---------------------------------------------------------------- NVFP4
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two f16 fragment halves from the E2M1 codes at bits [SH, SH+4) and
// [SH+16, SH+20) of w (SH = 0 or 4): magnitude bits to 9..11, sign to 15,
// i.e. the code's value times 2^-14.
template <int SH>
__device__ __forceinline__ uint32_t e2m1x2_f16(uint32_t w) {
  static_assert(SH == 0 || SH == 4, "nibble offset");
  // the two moves as one multiply-add (the fields are disjoint, so + is |),
  // which runs on the FMA pipe beside the integer pipe's masks
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;"
      : "=r"(r)
      : "r"(w & (0x00080008u << SH)), "n"(1u << (12 - SH)), "r"((w << (9 - SH)) & 0x0E000E00u));
  return r;
}

__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float f[4]) {
  const __half2 lo(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3));
  const __half2 hi(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3));
  const float2 a = __half22float2(lo), b = __half22float2(hi);
  f[0] = a.x, f[1] = a.y, f[2] = b.x, f[3] = b.y;
}

// Shared-memory order of the 16 channels of a block: position p of the
// tensor-core k index holds channel kNvPerm[p], matching the nibbles a lane
// takes from its code word (lane t, word (t >> 1) of the block, byte t & 1
// and byte (t & 1) + 2, low nibbles for k 2t, 2t+1, high nibbles for 2t+8,
// 2t+9).
// (p = k3 k2 k1 k0 in bits -> channel k2 k0 k1 k3: 0 4 2 6 8 12 10 14 1 5 3 7 9 13 11 15)
__host__ __device__ constexpr int nv_perm(int p) {
  return (((p >> 2) & 1) << 3) | ((p & 1) << 2) | (((p >> 1) & 1) << 1) | ((p >> 3) & 1);
}

// One warp quantises one row of nb 16-value blocks to NVFP4 and stores the
// values E2M1(q) * S_b (exact in f16) in tensor-core k order at out[16 nb];
// returns the row's global.  load(b, v) fills v with block b of the row.
// The same fp32 operations as the format's quantiser decide every code.
template <class Load>
__device__ __forceinline__ float nvfp4_row_f16(Load load, int nb, uint16_t *out) {
  const int lane = threadIdx.x & 31;
  float amax = 0.f;
  for (int b = lane; b < nb; b += 32) {
    float v[16];
    load(b, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float G = amax == 0.f ? 1.0f : __fdiv_rn(amax, 2688.0f);
  for (int b = lane; b < nb; b += 32) {
    float v[16];
    load(b, v);
    float bmax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
    const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(__fdiv_rn(bmax, __fmul_rn(6.0f, G)),
                                                        __NV_SATFINITE, __NV_E4M3);
    const float sb = __half2float(__half(__nv_cvt_fp8_to_halfraw(s8, __NV_E4M3)));
    const float scale = __fmul_rn(sb, G);
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const __nv_fp4_storage_t c = __nv_cvt_float_to_fp4(__fdiv_rn(v[i], scale), __NV_E2M1,
                                                         cudaRoundNearest);
      const float e = __half2float(__half(__nv_cvt_fp4_to_halfraw(c, __NV_E2M1)));
      q[i] = sb == 0.f ? 0.f : __fmul_rn(e, sb);
    }
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = (uint32_t)__half_as_ushort(__float2half_rn(q[nv_perm(2 * i)])) |
             ((uint32_t)__half_as_ushort(__float2half_rn(q[nv_perm(2 * i + 1)])) << 16);
    uint4 *dst = reinterpret_cast<uint4 *>(out + 16 * b);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  return G;
}

// Cooperative form of nvfp4_row_f16 for values already in registers: the
// participating threads (index t of nthreads, a multiple of 32) hold channel
// pairs P = t + nthreads * i (i < MAXP) of `rows` rows of K channels, pair P
// being row P / (K/2), channels 2 (P % (K/2)) and + 1, in hv[i].  A 16-value
// block is 8 consecutive lanes, a warp's 32 pairs lie in one row.  rowmax
// [rows] (shared, zeroed by the caller before the last barrier) collects
// the row maxima; between the two halves the caller's barrier `sync` runs.
// Same fp32 decisions as nvfp4_row_f16.
template <int MAXP, class Sync>
__device__ __forceinline__ void nvfp4_pairs_f16(const float2 (&hv)[MAXP], int rows, int K, int t,
                                                int nthreads, unsigned int *rowmax, float *Gout,
                                                uint16_t *out, Sync sync) {
  const int lane = threadIdx.x & 31, half = K / 2, total = rows * half;
  float bmax[MAXP];
#pragma unroll
  for (int i = 0; i < MAXP; ++i) {
    const int P = t + nthreads * i;
    float m = P < total ? fmaxf(fabsf(hv[i].x), fabsf(hv[i].y)) : 0.f;
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    bmax[i] = m;
    float r = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, 16));
    if (lane == 0 && P < total) atomicMax(&rowmax[P / half], __float_as_uint(r));
  }
  sync();
#pragma unroll
  for (int i = 0; i < MAXP; ++i) {
    const int P = t + nthreads * i;
    if (P >= total) continue;
    const int n = P / half, c2 = 2 * (P % half);  // first channel of the pair
    const float amax = __uint_as_float(rowmax[n]);
    const float G = amax == 0.f ? 1.0f : __fdiv_rn(amax, 2688.0f);
    if (c2 == 0) Gout[n] = G;
    const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(__fdiv_rn(bmax[i], __fmul_rn(6.0f, G)),
                                                        __NV_SATFINITE, __NV_E4M3);
    const float sb = __half2float(__half(__nv_cvt_fp8_to_halfraw(s8, __NV_E4M3)));
    const float scale = __fmul_rn(sb, G);
    const float v2[2] = {hv[i].x, hv[i].y};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const __nv_fp4_storage_t c = __nv_cvt_float_to_fp4(__fdiv_rn(v2[j], scale), __NV_E2M1,
                                                         cudaRoundNearest);
      const float e = __half2float(__half(__nv_cvt_fp4_to_halfraw(c, __NV_E2M1)));
      const float q = sb == 0.f ? 0.f : __fmul_rn(e, sb);
      // tensor-core k order inside the 16-channel block (inverse of nv_perm)
      const int ch = (c2 + j) & 15;
      const int kap = ((ch & 1) << 3) | (((ch >> 3) & 1) << 2) | (((ch >> 1) & 1) << 1) | ((ch >> 2) & 1);
      out[(size_t)n * K + ((c2 + j) & ~15) + kap] = __half_as_ushort(__float2half_rn(q));
    }
  }
}

// One warp, one 64-channel chunk g of NMAT NVFP4 strips (K channels each)
// against up to 16 activation rows act[n][ld] (f16 in tensor-core k order):
// acc += S_b * (sum over the block of code * 2^-14 * activation), block by
// block.  The A fragments are built once for both token blocks.
template <int NB, int NMAT>
__device__ __forceinline__ void fp4_chunk_mma(const uint8_t *const (&strip)[NMAT], int K, int g,
                                              const uint16_t *act, int ld, const int *tok_of,
                                              int ntok, float acc[NMAT][2][4]) {
  const int lane = threadIdx.x & 31, gi = lane >> 2, t4 = lane & 3;
  const int sh = 8 * (t4 & 1);
  const int rowoff = gi * (K / 2) + 128 * (g >> 2) + 4 * (t4 >> 1);
  uint32_t af[NMAT][4][4];
  float slo[NMAT][4], shi[NMAT][4];
#pragma unroll
  for (int m = 0; m < NMAT; ++m) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int off = rowoff + ((((2 * g + (j >> 1)) & 7) ^ (gi & 7)) << 4) + 8 * (j & 1);
      // this lane's bytes (t & 1) and (t & 1) + 2 of the word, moved to bytes 0 and 2
      const uint32_t wlo = *reinterpret_cast<const uint32_t *>(strip[m] + off) >> sh;
      const uint32_t whi = *reinterpret_cast<const uint32_t *>(strip[m] + off + 8 * (K / 2)) >> sh;
      af[m][j][0] = e2m1x2_f16<0>(wlo);
      af[m][j][1] = e2m1x2_f16<0>(whi);
      af[m][j][2] = e2m1x2_f16<4>(wlo);
      af[m][j][3] = e2m1x2_f16<4>(whi);
    }
    const uint8_t *sc = strip[m] + 8 * K + 64 * g;
    e4m3x4_to_f32(*reinterpret_cast<const uint32_t *>(sc + 4 * gi), slo[m]);
    e4m3x4_to_f32(*reinterpret_cast<const uint32_t *>(sc + 4 * (gi + 8)), shi[m]);
  }
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int n = nb * 8 + gi;
    const bool live = n < ntok;
    const uint16_t *arow = act + (size_t)(live ? tok_of[n] : 0) * ld + 64 * g + 2 * t4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t b0 = live ? *reinterpret_cast<const uint32_t *>(arow + 16 * j) : 0u;
      const uint32_t b1 = live ? *reinterpret_cast<const uint32_t *>(arow + 16 * j + 8) : 0u;
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        mma_f16_16816(d, af[m][j], b0, b1);
        acc[m][nb][0] = __fmaf_rn(slo[m][j], d[0], acc[m][nb][0]);
        acc[m][nb][1] = __fmaf_rn(slo[m][j], d[1], acc[m][nb][1]);
        acc[m][nb][2] = __fmaf_rn(shi[m][j], d[2], acc[m][nb][2]);
        acc[m][nb][3] = __fmaf_rn(shi[m][j], d[3], acc[m][nb][3]);
      }
    }
  }
}

template <int NB, int NMAT>
__device__ __forceinline__ void fp4_warp_chunks(const uint8_t *const (&strip)[NMAT], int K,
                                                int first, int step, const uint16_t *act, int ld,
                                                const int *tok_of, int ntok,
                                                float acc[NMAT][2][4]) {
  for (int g = first; g < K / 64; g += step)
    fp4_chunk_mma<NB, NMAT>(strip, K, g, act, ld, tok_of, ntok, acc);
}

}  // namespace moe
