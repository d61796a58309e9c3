// nvfp4.cuh -- NVFP4 device layout shared by the format, decode and prefill
// kernels.
//
// One [N][K] matrix is stored as N/16 strips (device strip order as for int4:
// a gate/up matrix alternates gate strip i and up strip i).  A strip is
//   codes  [16][K/2] bytes: logical byte b of row r holds channel 2b in its
//          low nibble and channel 2b + 1 in its high nibble, and sits at
//          nvfp4_code_pos(r, b): inside each 128-byte run of the row the
//          16-byte pieces are XOR-permuted by (r & 7), the 128-byte swizzle
//          that the tensor cores read from shared memory, so a plain copy of
//          rows x 128 bytes is a ready operand tile, and the eight rows r & 7
//          of a strip put the same logical byte in eight different banks;
//   scales [K/64][16][4] E4M3 bytes: for each 64 channels, the 4 block
//          scales (16 channels each) of the 16 rows, row after row;
// so 9K bytes per strip, 4.5 bits per weight.  K % 256 == 0.
#pragma once

#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

__host__ __device__ inline size_t nvfp4_strip_bytes(int K) { return (size_t)9 * (size_t)K; }

// Byte offset, inside a strip's code array, of logical byte b of row r.
__host__ __device__ inline int nvfp4_code_pos(int r, int b, int K) {
  return r * (K / 2) + (b & ~127) + ((((b >> 4) & 7) ^ (r & 7)) << 4) + (b & 15);
}
// Byte offset, inside a strip's scale array, of row r's scale for channels
// [16 blk, 16 blk + 16).
__host__ __device__ inline int nvfp4_scale_pos(int r, int blk) {
  return (blk >> 2) * 64 + r * 4 + (blk & 3);
}

#ifdef __CUDACC__
__device__ __forceinline__ float e4m3_to_f32(uint8_t s) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)s, __NV_E4M3)));
}
#endif

}  // namespace moe
