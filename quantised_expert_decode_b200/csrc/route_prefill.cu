// Router for prefill chunks (T > 8 or bf16 activations).
#include "common.cuh"

namespace qmoe {

size_t route_prefill_ws_bytes(int T, int E) { return (((size_t)T * E * sizeof(double) + 255) & ~(size_t)255) + 256; }

qmoe_status route_prefill(const float *, const float *, const void *, int, int, int, int, int, int32_t *, float *,
                          void *, size_t, int32_t *, cudaStream_t) {
  return QMOE_ERR_UNSUPPORTED;
}

}  // namespace qmoe
