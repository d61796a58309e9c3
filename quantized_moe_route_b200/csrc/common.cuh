// common.cuh -- shared host/device helpers of libmoe (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoe is written for sm_100a (B200) only"
#endif

namespace moe {

// ---------------------------------------------------------------- host side
void set_cuda_error(cudaError_t e);
moe_status launch_status();  // checks cudaGetLastError after a launch

inline cudaStream_t as_stream(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel on the stream drains, so it calls grid_dep_wait()
// before it reads anything earlier work wrote.  Returns the launch status.
template <typename... KArgs, typename... Args>
inline moe_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Device error word (one per device, cleared by moe_device_error).
enum : int {
  DEVERR_NONE = 0,
  DEVERR_DECODE_H_WAIT = 0x101,   // decode: down projection waited too long for h
  DEVERR_DECODE_ROUTER_WAIT = 0x102,  // decode: routing waited too long for a logit
  DEVERR_PREFILL_WAIT = 0x201,    // prefill: a pipeline barrier wait gave up
};
int *device_error_word();  // device address of the word on the current device

// Layout of one packed int4 block: 16 rows x 64 input channels.
constexpr int kBlkRows = 16;
constexpr int kGroup = 64;
constexpr int kBlkCodeBytes = 512;
constexpr int kBlkBytes = 576;

__host__ __device__ inline size_t w4_packed_bytes(int N, int K) {
  return (size_t)(N / kBlkRows) * (size_t)(K / kGroup) * kBlkBytes;
}

// Device strip index of canonical row n (a multiple of 16).  Gate/up:
// canonical rows [0, F) gate, [F, 2F) up; device strips alternate gate, up.
__host__ __device__ inline int w4_strip_of_row(int n, int N, int kind) {
  if (kind == MOE_W4_GATE_UP) {
    int F = N / 2;
    return n < F ? 2 * (n / kBlkRows) : 2 * ((n - F) / kBlkRows) + 1;
  }
  return n / kBlkRows;
}
__host__ __device__ inline int w4_row_of_strip(int s, int N, int kind) {
  if (kind == MOE_W4_GATE_UP) {
    int F = N / 2;
    return (s & 1) ? F + (s >> 1) * kBlkRows : (s >> 1) * kBlkRows;
  }
  return s * kBlkRows;
}

// Position of canonical (row r in 0..15, channel c in 0..63) of a block:
// lane (0..31), word (0..3) and nibble shift inside the word.  The word of
// lane l = 4*g + t for k16-step j holds, nibble by nibble (shift 0, 4, 8, ...,
// 28): (g, 16j+2t), (g+8, 16j+2t), (g, 16j+2t+8), (g+8, 16j+2t+8),
//       (g, 16j+2t+1), (g+8, 16j+2t+1), (g, 16j+2t+9), (g+8, 16j+2t+9).
// Masking the word with 0x000F000F after a right shift of 0, 4, 8 or 12 gives
// the bf16x2 pairs of the m16n8k16 A fragment registers a0a1, a2a3, a4a5, a6a7.
__host__ __device__ inline void w4_block_pos(int r, int c, int *lane, int *word, int *shift) {
  int g = r & 7, hi_row = r >> 3;
  int j = c >> 4, cc = c & 15;
  int hi_k = cc >> 3, t = (cc & 7) >> 1, odd = cc & 1;
  *lane = 4 * g + t;
  *word = j;
  *shift = 16 * odd + 8 * hi_k + 4 * hi_row;
}

// ---------------------------------------------------------------- device side
#ifdef __CUDACC__

// Programmatic dependent launch: wait until the previous kernel on the
// stream has completed and its writes are visible; let the next kernel on the
// stream begin launching (it still waits for this one before reading).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// mbarrier (shared memory, CTA scope)
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and leaves the barrier alone) after `limit`
// failed polls.  Each try_wait itself suspends for a hardware-chosen time.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Bounded wait for warps that have nothing else to do: each poll suspends
// the thread until the phase completes or about hint_ns have passed, so a
// waiting warp takes few issue slots.  At most `limit` polls.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t limit,
                                                uint32_t hint_ns = 10000u) {
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Order this thread's generic-proxy shared-memory accesses before later
// async-proxy accesses (bulk/TMA copies, tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier (no
// multicast).  Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_g2s_evict_first(void *dst, const void *src, uint32_t bytes,
                                                     uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Legacy warp-level MMA used by the decode kernel as its dot-product engine:
// D[16x8] (fp32) = A[16x16] (bf16, row) * B[16x8] (bf16, col) + C.
__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte asynchronous global -> shared copy (no register staging).
__device__ __forceinline__ void cp_async_16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(int *p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}
__device__ __forceinline__ float f16_bits_to_f32(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}
// bf16 pair {lo, hi} (lo in the low half), each rounded to nearest even
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// Shared-memory accesses by 32-bit shared-window address.
__device__ __forceinline__ void sts_b32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t lds_b32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

#endif  // __CUDACC__

}  // namespace moe
