// Host-side helpers of libqmoe: status mapping, device queries, launch counter.
#include <atomic>

#include "common.cuh"

namespace qmoe {

static std::atomic<uint64_t> g_launches{0};

void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

qmoe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QMOE_OK : QMOE_ERR_CUDA; }

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

size_t max_smem_optin() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return (size_t)n;
}

}  // namespace qmoe

extern "C" uint64_t qmoe_launch_count(void) { return qmoe::g_launches.load(); }

extern "C" const char *qmoe_status_string(qmoe_status s) {
  switch (s) {
    case QMOE_OK: return "ok";
    case QMOE_ERR_INVALID_ARG: return "invalid argument";
    case QMOE_ERR_GEOMETRY: return "expert geometry mismatch";
    case QMOE_ERR_UNSUPPORTED: return "unsupported shape or format";
    case QMOE_ERR_WORKSPACE: return "workspace too small";
    case QMOE_ERR_CUDA: return "CUDA runtime error";
    case QMOE_ERR_TIMEOUT: return "device wait exceeded its budget";
    case QMOE_ERR_DEVICE_STATUS: return "invalid routed expert index seen on the device";
    case QMOE_ERR_RANGE: return "activation too large for the exact decode sums";
  }
  return "unknown status";
}

extern "C" qmoe_status qmoe_read_status(const int32_t *dev_status) {
  if (!dev_status) return QMOE_ERR_INVALID_ARG;
  int32_t v = 0;
  if (cudaMemcpy(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return QMOE_ERR_CUDA;
  switch (v) {
    case qmoe::DEV_OK: return QMOE_OK;
    case qmoe::DEV_TIMEOUT: return QMOE_ERR_TIMEOUT;
    case qmoe::DEV_RANGE: return QMOE_ERR_RANGE;
    default: return QMOE_ERR_DEVICE_STATUS;
  }
}
