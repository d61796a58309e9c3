// prefill.cu -- grouped expert FFN on the tensor cores (tcgen05).
#include "common.cuh"

using namespace moe;

extern "C" MOE_API size_t moe_prefill_workspace_bytes(int rows, int F) {
  if (rows <= 0 || F <= 0) return 0;
  return (size_t)rows * F * 2 + 4096;
}

extern "C" MOE_API moe_status moe_ffn_grouped_prefill(const moe_w4_layer *layer,
                                                      const uint16_t *x_perm,
                                                      const int32_t *offsets, int rows,
                                                      uint16_t *y_perm, void *ws, size_t ws_bytes,
                                                      moe_stream_t stream) {
  (void)layer; (void)x_perm; (void)offsets; (void)rows; (void)y_perm; (void)ws; (void)ws_bytes;
  (void)stream;
  return MOE_ERR_UNSUPPORTED_SHAPE;
}
