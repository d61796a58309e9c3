// decode_items.cuh -- the int4 work of one warp on one decode work item, with
// every shared-memory address formed once per item (32-bit shared-window
// addresses advanced by a constant stride per group).
//
// A warp takes the groups g0, g0 + step, ... (ngw of them) of NMAT packed
// int4 matrices of 16 rows (blocks of 576 bytes: codes in the lanes' fragment
// order, then 16 x {f16 scale, f16 min}), against up to 16 activation rows
// held as bf16 [row][ld] in w4_kpos order with their 64-channel group sums.
// Per group and matrix: the four k16 A fragments from one 16-byte load (the
// bf16 values 128 + q), four m16n8k16 MMAs per token block, and the fold
//   acc += s D + (m - 128 s) X
// -- the same operations, in the same order for every accumulator, as
// group_mma, so the results are the same bits.
#pragma once
#include "decode_common.cuh"

namespace moe {

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// wa[m]: shared address of matrix m's block of group 0 (blocks 576 bytes
// apart); act_s / gsum_s: shared addresses of the activation rows and of
// their group sums; tok_of[n]: activation row of token column n.
template <int NB, int NMAT>
__device__ __forceinline__ void w4_item(const uint32_t (&wa)[NMAT], int g0, int step, int ngw,
                                        uint32_t act_s, int ld, const int *tok_of, int ntok,
                                        uint32_t gsum_s, int gsum_ld, float acc[NMAT][2][4]) {
  const int lane = threadIdx.x & 31, gi = lane >> 2, t4 = lane & 3;
  const uint32_t wstep = (uint32_t)step * kBlkBytes, astep = (uint32_t)step * 128u, sstep = (uint32_t)step * 4u;
  uint32_t wc[NMAT];
#pragma unroll
  for (int m = 0; m < NMAT; ++m) wc[m] = wa[m] + (uint32_t)g0 * kBlkBytes;
  uint32_t ar[NB], ga[NB], gb[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int n = nb * 8 + gi, na = nb * 8 + 2 * t4;
    ar[nb] = act_s + 2u * (uint32_t)(tok_of[n < ntok ? n : 0] * ld + 64 * g0 + 16 * t4);
    ga[nb] = gsum_s + 4u * (uint32_t)(tok_of[na < ntok ? na : 0] * gsum_ld + g0);
    gb[nb] = gsum_s + 4u * (uint32_t)(tok_of[na + 1 < ntok ? na + 1 : 0] * gsum_ld + g0);
  }
#pragma unroll 2
  for (int i = 0; i < ngw; ++i) {
    uint32_t af[NMAT][4][4];
    GroupAffine aff[NMAT];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      const uint4 cw = lds_u4(wc[m] + 16u * lane);
      w4_frag(cw.x, af[m][0]);
      w4_frag(cw.y, af[m][1]);
      w4_frag(cw.z, af[m][2]);
      w4_frag(cw.w, af[m][3]);
      const uint32_t lo = lds_b32(wc[m] + kBlkCodeBytes + 4u * gi);
      const uint32_t hi = lds_b32(wc[m] + kBlkCodeBytes + 4u * (gi + 8));
      aff[m].s0 = f16_bits_to_f32((uint16_t)(lo & 0xFFFFu));
      aff[m].s1 = f16_bits_to_f32((uint16_t)(hi & 0xFFFFu));
      aff[m].c0 = __fmaf_rn(-128.f, aff[m].s0, f16_bits_to_f32((uint16_t)(lo >> 16)));
      aff[m].c1 = __fmaf_rn(-128.f, aff[m].s1, f16_bits_to_f32((uint16_t)(hi >> 16)));
      wc[m] += wstep;
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const uint4 q0 = lds_u4(ar[nb]), q1 = lds_u4(ar[nb] + 16u);
      const float xa = lds_f32(ga[nb]), xb = lds_f32(gb[nb]);
      const uint32_t b[4][2] = {{q0.x, q0.y}, {q0.z, q0.w}, {q1.x, q1.y}, {q1.z, q1.w}};
      const float xs[4] = {xa, xb, xa, xb};
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_bf16_16816(d, af[m][j], b[j][0], b[j][1]);
        fold(acc[m][nb], d, xs, aff[m]);
      }
      ar[nb] += astep;
      ga[nb] += sstep;
      gb[nb] += sstep;
    }
  }
}

// acq_rel atomic add at GPU scope: releases this thread's (and, through a
// preceding barrier, its CTA's) earlier writes and acquires those released
// by the earlier adds on the same word.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int *p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

}  // namespace moe
