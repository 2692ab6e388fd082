// Router for decode batches (T <= 8): float64 GEMV over fp32 weights, top-k with
// ties to the lower expert index, renormalised gates; optionally preceded by
// the residual RMSNorm of the previous layer's output.
#include <mutex>

#include "common.cuh"
#include "route_common.cuh"

namespace qmoe {
namespace {

constexpr int RT_THREADS = 128;  // 4 warps, one router row per warp at a time
constexpr int RT_MAXT = 8;
constexpr int RT_PREFETCH = 16;  // float4 per lane held across the dependency wait

struct RouteArgs {
  const float *Wr;
  const float *bias;
  const float *x;
  const float *y;      // residual input (RESID only)
  float *x_out;        // normalised activations (RESID only)
  float eps;
  int T, H, E, k;
  int32_t *idx;
  float *gate;
  double *logits;      // workspace [T, E]
  unsigned *ticket;    // workspace
  int32_t *status;
};

template <bool RESID>
__global__ void __launch_bounds__(RT_THREADS) route_decode_kernel(RouteArgs a) {
  extern __shared__ float4 xs4[];  // [T][H/4]
  __shared__ float inv_rms[RT_MAXT];
  __shared__ unsigned is_last;
  __shared__ TopkScratch topk_sc[RT_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.T, H = a.H, E = a.E, H4 = H / 4;

  // This warp's router row does not depend on the previous kernel: fetch it
  // into registers (H <= 2048 entirely) before waiting for that kernel.
  const int e_row = blockIdx.x * (RT_THREADS / 32) + warp;
  float4 wpre[RT_PREFETCH];
  if (e_row < E) {
    const float4 *w4 = reinterpret_cast<const float4 *>(a.Wr + (size_t)e_row * H);
#pragma unroll
    for (int j = 0; j < RT_PREFETCH; ++j)
      if (lane + 32 * j < H4) wpre[j] = __ldg(w4 + lane + 32 * j);
  }
  pdl_wait();
  pdl_launch_dependents();

  const float4 *x4 = reinterpret_cast<const float4 *>(a.x);
  const float4 *y4 = reinterpret_cast<const float4 *>(a.y);
  for (int i = tid; i < T * H4; i += RT_THREADS) {
    float4 v = x4[i];
    if (RESID) {
      float4 w = y4[i];
      v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
    }
    xs4[i] = v;
  }
  __syncthreads();
  if (RESID) {
    for (int t = warp; t < T; t += RT_THREADS / 32) {
      double ss = 0.0;
      for (int j = lane; j < H4; j += 32) {
        float4 v = xs4[t * H4 + j];
        ss += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
      }
      ss = warp_sum_d(ss);
      if (lane == 0) inv_rms[t] = (float)(1.0 / sqrt(ss / (double)H + (double)a.eps));
    }
    __syncthreads();
    float4 *xo4 = reinterpret_cast<float4 *>(a.x_out);
    for (int i = tid; i < T * H4; i += RT_THREADS) {
      float s = inv_rms[i / H4];
      float4 v = xs4[i];
      v.x *= s; v.y *= s; v.z *= s; v.w *= s;
      xs4[i] = v;
      if (blockIdx.x == 0) xo4[i] = v;
    }
    __syncthreads();
  }

  // logits: one warp per router row, float64 accumulation of exact products
  if (e_row < E) {
    const float4 *w4 = reinterpret_cast<const float4 *>(a.Wr + (size_t)e_row * H);
    const double b = a.bias ? (double)a.bias[e_row] : 0.0;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
      double s = 0.0;
#pragma unroll
      for (int jj = 0; jj < RT_PREFETCH; ++jj) {
        const int j = lane + 32 * jj;
        if (j < H4) {
          const float4 w = wpre[jj], v = xs4[t * H4 + j];
          s = fma((double)w.x, (double)v.x, s);
          s = fma((double)w.y, (double)v.y, s);
          s = fma((double)w.z, (double)v.z, s);
          s = fma((double)w.w, (double)v.w, s);
        }
      }
      for (int j = lane + 32 * RT_PREFETCH; j < H4; j += 32) {
        const float4 w = __ldg(w4 + j), v = xs4[t * H4 + j];
        s = fma((double)w.x, (double)v.x, s);
        s = fma((double)w.y, (double)v.y, s);
        s = fma((double)w.z, (double)v.z, s);
        s = fma((double)w.w, (double)v.w, s);
      }
      s = warp_sum_d(s);
      if (lane == 0) a.logits[(size_t)t * E + e_row] = s + b;
    }
  }

  // the last CTA to finish selects the experts of every token
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1u) ? 1u : 0u;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int t = warp; t < T; t += RT_THREADS / 32)
    warp_topk_gates(a.logits + (size_t)t * E, E, a.k, a.idx + t * a.k, a.gate + t * a.k, &topk_sc[warp]);
  __syncthreads();
  if (tid == 0) atomicExch(a.ticket, 0u);
}

__global__ void rmsnorm_residual_kernel(const float *x, const float *y, float eps, float *out, int H) {
  __shared__ double part[32];
  __shared__ float inv;
  const int t = blockIdx.x;
  const float *xr = x + (size_t)t * H;
  const float *yr = y + (size_t)t * H;
  double ss = 0.0;
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    float z = xr[h] + yr[h];
    ss += (double)z * z;
  }
  ss = warp_sum_d(ss);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < blockDim.x / 32 ? part[threadIdx.x] : 0.0;
    v = warp_sum_d(v);
    if (threadIdx.x == 0) inv = (float)(1.0 / sqrt(v / (double)H + (double)eps));
  }
  __syncthreads();
  for (int h = threadIdx.x; h < H; h += blockDim.x) out[(size_t)t * H + h] = (xr[h] + yr[h]) * inv;
}

size_t decode_ws_bytes(int T, int E) { return (((size_t)T * E * sizeof(double) + 255) & ~(size_t)255) + 256; }

qmoe_status launch_route_decode(const RouteArgs &a, bool resid, cudaStream_t s) {
  size_t smem = (size_t)a.T * a.H * sizeof(float);
  int grid = (a.E + RT_THREADS / 32 - 1) / (RT_THREADS / 32);
  const void *fn = resid ? (const void *)route_decode_kernel<true> : (const void *)route_decode_kernel<false>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMOE_ERR_CUDA;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(RT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = resid ? cudaLaunchKernelEx(&cfg, route_decode_kernel<true>, a)
                        : cudaLaunchKernelEx(&cfg, route_decode_kernel<false>, a);
  note_launch();
  return cuda_status(e);
}

}  // namespace

// Shared with the prefill router (route_prefill.cu).
qmoe_status route_prefill(const float *Wr, const float *bias, const void *x, int x_dtype, int T, int H, int E, int k,
                          int32_t *idx, float *gate, void *ws, size_t ws_bytes, int32_t *status, cudaStream_t s);
size_t route_prefill_ws_bytes(int T, int E);

}  // namespace qmoe

using namespace qmoe;

static qmoe_status check_route_common(const float *Wr, int T, int H, int E, int k, const int32_t *idx,
                                      const float *gate, const void *ws, const int32_t *status) {
  if (!Wr || !idx || !gate || !ws || !status) return QMOE_ERR_INVALID_ARG;
  if (!aligned16(Wr) || !aligned16(ws)) return QMOE_ERR_INVALID_ARG;
  if (T < 1 || H < 128 || E < 1 || k < 1) return QMOE_ERR_INVALID_ARG;
  if (H % 128) return QMOE_ERR_UNSUPPORTED;
  if (k > 16 || k > E || E > 1024) return QMOE_ERR_UNSUPPORTED;
  return QMOE_OK;
}

extern "C" size_t qmoe_route_workspace_bytes(int T, int E) {
  if (T <= 0 || E <= 0) return 0;
  // T <= 8 with bf16 x runs the prefill router, so cover both
  if (T <= RT_MAXT) return decode_ws_bytes(T, E) > route_prefill_ws_bytes(T, E) ? decode_ws_bytes(T, E)
                                                                                : route_prefill_ws_bytes(T, E);
  return route_prefill_ws_bytes(T, E);
}

extern "C" qmoe_status qmoe_route(const float *Wr, const float *bias, const void *x, int x_dtype, int T, int H, int E,
                                  int k, int32_t *idx, float *gate, void *workspace, size_t workspace_bytes,
                                  int32_t *dev_status, qmoe_stream_t stream) {
  qmoe_status st = check_route_common(Wr, T, H, E, k, idx, gate, workspace, dev_status);
  if (st != QMOE_OK) return st;
  if (!x || !aligned16(x)) return QMOE_ERR_INVALID_ARG;
  if (x_dtype != QMOE_F32 && x_dtype != QMOE_BF16) return QMOE_ERR_INVALID_ARG;
  if (workspace_bytes < qmoe_route_workspace_bytes(T, E)) return QMOE_ERR_WORKSPACE;
  if (T > RT_MAXT || x_dtype == QMOE_BF16)
    return route_prefill(Wr, bias, x, x_dtype, T, H, E, k, idx, gate, workspace, workspace_bytes, dev_status,
                         (cudaStream_t)stream);
  RouteArgs a{};
  a.Wr = Wr;
  a.bias = bias;
  a.x = static_cast<const float *>(x);
  a.T = T; a.H = H; a.E = E; a.k = k;
  a.idx = idx;
  a.gate = gate;
  a.logits = static_cast<double *>(workspace);
  a.ticket = reinterpret_cast<unsigned *>(static_cast<char *>(workspace) + decode_ws_bytes(T, E) - 256);
  a.status = dev_status;
  return launch_route_decode(a, false, (cudaStream_t)stream);
}

extern "C" qmoe_status qmoe_residual_route(const float *x_in, const float *y, float eps, float *x_out, const float *Wr,
                                           const float *bias, int T, int H, int E, int k, int32_t *idx, float *gate,
                                           void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                           qmoe_stream_t stream) {
  qmoe_status st = check_route_common(Wr, T, H, E, k, idx, gate, workspace, dev_status);
  if (st != QMOE_OK) return st;
  if (!x_in || !y || !x_out || !aligned16(x_in) || !aligned16(y) || !aligned16(x_out)) return QMOE_ERR_INVALID_ARG;
  if (x_out == x_in || x_out == y) return QMOE_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return QMOE_ERR_INVALID_ARG;
  if (T > RT_MAXT) return QMOE_ERR_UNSUPPORTED;
  if (workspace_bytes < qmoe_route_workspace_bytes(T, E)) return QMOE_ERR_WORKSPACE;
  RouteArgs a{};
  a.Wr = Wr;
  a.bias = bias;
  a.x = x_in;
  a.y = y;
  a.x_out = x_out;
  a.eps = eps;
  a.T = T; a.H = H; a.E = E; a.k = k;
  a.idx = idx;
  a.gate = gate;
  a.logits = static_cast<double *>(workspace);
  a.ticket = reinterpret_cast<unsigned *>(static_cast<char *>(workspace) + decode_ws_bytes(T, E) - 256);
  a.status = dev_status;
  return launch_route_decode(a, true, (cudaStream_t)stream);
}

// ----------------------------------------------------------- fixed scratch --
// The decode router for callers that cannot allocate device memory for a
// workspace: a host program that owns only its input/output buffers and has
// no allocator, or a serving loop that may not call into one (an allocation
// can synchronise the device). The scratch lives in one fixed device array
// per device, so concurrent calls on one device race for it.
namespace qmoe {
namespace {

constexpr size_t FIXED_LOGITS_BYTES = (size_t)QMOE_ROUTE_FIXED_MAX_T * QMOE_ROUTE_FIXED_MAX_E * sizeof(double);
static_assert(QMOE_ROUTE_FIXED_SCRATCH_BYTES == FIXED_LOGITS_BYTES + 256, "fixed scratch layout");

// [0, FIXED_LOGITS_BYTES): float64 logits; then the 256-byte ticket block,
// which must start at zero (each completed call leaves it at zero).
__device__ __align__(256) unsigned char g_route_scratch[QMOE_ROUTE_FIXED_SCRATCH_BYTES];

constexpr int FIXED_MAX_DEVICES = 64;
std::mutex g_fixed_mutex;
void *g_fixed_ptr[FIXED_MAX_DEVICES];

// First call on a device: look up the array's address and zero it
// (synchronous; no allocation). Later calls reuse the address.
qmoe_status fixed_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QMOE_ERR_CUDA;
  if (dev < 0 || dev >= FIXED_MAX_DEVICES) return QMOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_fixed_mutex);
  if (!g_fixed_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return QMOE_ERR_CUDA;
    if (cudaMemset(p, 0, QMOE_ROUTE_FIXED_SCRATCH_BYTES) != cudaSuccess) return QMOE_ERR_CUDA;
    g_fixed_ptr[dev] = p;
  }
  *out = g_fixed_ptr[dev];
  return QMOE_OK;
}

}  // namespace
}  // namespace qmoe

extern "C" qmoe_status qmoe_route_fixed(const float *Wr, const float *bias, const float *x, int T, int H, int E, int k,
                                        int32_t *idx, float *gate, int32_t *dev_status, qmoe_stream_t stream) {
  if (!Wr || !x || !idx || !gate || !dev_status) return QMOE_ERR_INVALID_ARG;
  if (!aligned16(Wr) || !aligned16(x)) return QMOE_ERR_INVALID_ARG;
  if (T < 1 || H < 128 || E < 1 || k < 1) return QMOE_ERR_INVALID_ARG;
  if (H % 128 || k > 16 || k > E) return QMOE_ERR_UNSUPPORTED;
  if (T > QMOE_ROUTE_FIXED_MAX_T || E > QMOE_ROUTE_FIXED_MAX_E) return QMOE_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  const qmoe_status st = fixed_scratch(&scratch);
  if (st != QMOE_OK) return st;
  RouteArgs a{};
  a.Wr = Wr;
  a.bias = bias;
  a.x = x;
  a.T = T; a.H = H; a.E = E; a.k = k;
  a.idx = idx;
  a.gate = gate;
  a.logits = static_cast<double *>(scratch);
  a.ticket = reinterpret_cast<unsigned *>(static_cast<char *>(scratch) + FIXED_LOGITS_BYTES);
  a.status = dev_status;
  return launch_route_decode(a, false, (cudaStream_t)stream);
}

extern "C" qmoe_status qmoe_rmsnorm_residual(const float *x_in, const float *y, float eps, float *x_out, int T, int H,
                                             qmoe_stream_t stream) {
  if (!x_in || !y || !x_out || T < 1 || H < 1) return QMOE_ERR_INVALID_ARG;
  if (!aligned16(x_in) || !aligned16(y) || !aligned16(x_out)) return QMOE_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return QMOE_ERR_INVALID_ARG;
  rmsnorm_residual_kernel<<<T, 256, 0, (cudaStream_t)stream>>>(x_in, y, eps, x_out, H);
  note_launch();
  return cuda_status(cudaGetLastError());
}
