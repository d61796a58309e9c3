// Test helper (not part of the library): a kernel that occupies one SM for a
// bounded number of clock cycles, holding as much shared memory as the caller
// asks for, so that no other large-shared-memory CTA fits on that SM
// meanwhile.  The wait ends by itself after `cycles` SM clock cycles.
#include <cuda_runtime.h>

__global__ void hold_kernel(long long cycles, int *done) {
  extern __shared__ unsigned char scratch[];
  const long long t0 = clock64();
  while (clock64() - t0 < cycles) __nanosleep(1000);
  if (threadIdx.x == 0) {
    scratch[0] = 1;
    *done = scratch[0];
  }
}

// One CTA of 32 threads with smem_bytes of dynamic shared memory on `stream`.
// Returns the CUDA error code (0 on success).
extern "C" int gpu_hold_sm(long long cycles, int smem_bytes, int *done, void *stream) {
  cudaError_t e = cudaFuncSetAttribute(hold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return (int)e;
  hold_kernel<<<1, 32, smem_bytes, static_cast<cudaStream_t>(stream)>>>(cycles, done);
  return (int)cudaGetLastError();
}
