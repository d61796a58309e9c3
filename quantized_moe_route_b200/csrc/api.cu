// api.cu -- status strings, CUDA error bookkeeping and the device error word.
#include <atomic>
#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace moe {

static thread_local char g_last_error[256] = "no error";

void set_cuda_error(cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
}

moe_status launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// One word per device; read and cleared by moe_device_error.
__device__ int g_device_error;

// The symbol's device address, looked up once per device (the lookup is not
// a stream operation, so it is also safe while a stream is being captured).
// Host threads may race on the first lookup; both find the same address.
int *device_error_word() {
  static std::atomic<int *> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  int *w = cached[dev].load(std::memory_order_acquire);
  if (!w) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    w = static_cast<int *>(p);
    cached[dev].store(w, std::memory_order_release);
  }
  return w;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

extern "C" MOE_API const char *moe_last_error_string(void) { return g_last_error; }

extern "C" MOE_API const char *moe_version(void) { return "moe-w4-b200 1"; }

extern "C" MOE_API moe_status moe_device_error(int *out, moe_stream_t stream) {
  if (!out) return MOE_ERR_INVALID_ARG;
  int *dev = device_error_word();
  if (!dev) {
    set_cuda_error(cudaGetLastError());
    return MOE_ERR_CUDA;
  }
  cudaError_t e = cudaMemcpyAsync(out, dev, sizeof(int), cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e == cudaSuccess && *out != 0) e = cudaMemsetAsync(dev, 0, sizeof(int), as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
