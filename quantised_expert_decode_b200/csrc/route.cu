// Router for decode batches (T <= 8): float64 router logits from exact
// fixed-point sums of 16-element slice partials, top-k with ties to the lower
// expert index, renormalised gates; optionally preceded by the residual
// RMSNorm of the previous layer's output. The arithmetic is the one of
// decode_canon.cuh, shared with the fused layer-stack kernel.
#include <mutex>

#include "common.cuh"
#include "decode_canon.cuh"
#include "route_common.cuh"

namespace qmoe {
namespace {

constexpr int RT_WARPS = 8;                // one router row per warp; one token per warp for the top-k
constexpr int RT_THREADS = 32 * RT_WARPS;
constexpr int RT_MAXT = 8;
constexpr int RT_PRE = 4;                  // slices per lane held in registers (all of H <= 2048)

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

// z = x (+ y) of every token sits in shared memory with one pad float after
// every 32: element h of token t at t * HP + h + h / 32 (HP = H + H / 32). A
// lane reads the 16 elements of one slice, lanes 16 elements apart; the pad
// spreads the 32 lanes of a warp over the 32 banks.
__host__ __device__ inline int route_hp(int H) { return H + H / 32; }
__device__ __forceinline__ int zpos(int h) { return h + (h >> 5); }
inline size_t route_smem_bytes(int T, int H) { return (size_t)T * route_hp(H) * 4; }

template <bool RESID>
__global__ void __launch_bounds__(RT_THREADS, 1) route_decode_kernel(RouteArgs a) {
  extern __shared__ __align__(16) float zs[];  // [T][HP], padded
  __shared__ double rinv_s[RT_MAXT];
  __shared__ float inv_s[RT_MAXT];
  __shared__ unsigned is_last;
  __shared__ int range_bad;
  __shared__ TopkScratch topk_sc[RT_WARPS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.T, H = a.H, E = a.E, nsl = H / canon::SLICE, HP = route_hp(H);
  const int e_row = blockIdx.x * RT_WARPS + warp;

  // This warp's router row does not depend on the previous kernel: fetch the
  // lane's slices (c = lane + 32 j) into registers before waiting for it.
  float4 wpre[RT_PRE][4];
  if (e_row < E) {
    const float4 *w4 = reinterpret_cast<const float4 *>(a.Wr + (size_t)e_row * H);
#pragma unroll
    for (int j = 0; j < RT_PRE; ++j) {
      const int c = lane + 32 * j;
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (c < nsl) wpre[j][m] = __ldg(w4 + c * 4 + m);
    }
  }
  if (tid == 0) range_bad = 0;
  pdl_wait();
  pdl_launch_dependents();

  // z = x (+ y) into the padded layout; eight float4 of each input in flight
  // per thread
  {
    const float4 *x4 = reinterpret_cast<const float4 *>(a.x);
    const float4 *y4 = reinterpret_cast<const float4 *>(a.y);
    const int n4 = T * H / 4, H4 = H / 4;
    constexpr int B = 8;
    for (int i0 = tid; i0 < n4; i0 += B * RT_THREADS) {
      float4 xv[B], yv[B];
#pragma unroll
      for (int u = 0; u < B; ++u) {
        const int i = i0 + u * RT_THREADS;
        if (i < n4) {
          xv[u] = __ldcg(x4 + i);
          if (RESID) yv[u] = __ldcg(y4 + i);
        }
      }
#pragma unroll
      for (int u = 0; u < B; ++u) {
        const int i = i0 + u * RT_THREADS;
        if (i < n4) {
          float4 v = xv[u];
          if (RESID) {
            v.x = __fadd_rn(v.x, yv[u].x); v.y = __fadd_rn(v.y, yv[u].y);
            v.z = __fadd_rn(v.z, yv[u].z); v.w = __fadd_rn(v.w, yv[u].w);
          }
          const int t = i / H4, h = 4 * (i % H4);
          float *zt = zs + (size_t)t * HP;
          zt[zpos(h)] = v.x; zt[zpos(h + 1)] = v.y; zt[zpos(h + 2)] = v.z; zt[zpos(h + 3)] = v.w;
        }
      }
    }
  }
  __syncthreads();
  if (RESID) {
    // sum of squares of every token (one warp per token), then 1 / rms
    for (int t = warp; t < T; t += RT_WARPS) {
      const float *zt = zs + (size_t)t * HP;
      const double ss = canon::warp_sumsq(
          [&](int c) { return canon::slice_sumsq([&](int i) { return zt[zpos(c * canon::SLICE + i)]; }); }, nsl);
      if (lane == 0) {
        const double r = canon::norm_rinv(ss, H, a.eps);
        rinv_s[t] = r;
        inv_s[t] = __double2float_rn(r);
      }
    }
    __syncthreads();
    if (blockIdx.x == 0) {
      float4 *xo4 = reinterpret_cast<float4 *>(a.x_out);
      const int H4 = H / 4;
      for (int i = tid; i < T * H4; i += RT_THREADS) {
        const int t = i / H4, h = 4 * (i % H4);
        const float s = inv_s[t];
        const float *zt = zs + (size_t)t * HP;
        xo4[i] = make_float4(__fmul_rn(zt[zpos(h)], s), __fmul_rn(zt[zpos(h + 1)], s), __fmul_rn(zt[zpos(h + 2)], s),
                             __fmul_rn(zt[zpos(h + 3)], s));
      }
    }
  } else {
    if (tid < RT_MAXT) rinv_s[tid] = 1.0;
    __syncthreads();
  }

  // logits: one warp per router row; slice partials split into exact integers
  if (e_row < E) {
    const float4 *w4 = reinterpret_cast<const float4 *>(a.Wr + (size_t)e_row * H);
    const double b = a.bias ? (double)a.bias[e_row] : 0.0;
    bool ok = true;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
      const float *zt = zs + (size_t)t * HP;
      long long hi = 0, lo = 0;
#pragma unroll
      for (int j = 0; j < RT_PRE; ++j) {
        const int c = lane + 32 * j;
        if (c < nsl) {
          const float *zc = zt + zpos(c * canon::SLICE);   // a slice never crosses a pad
          const double p = canon::slice_dot(
              [&](int i) {
                const float4 v = wpre[j][i >> 2];
                return (i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w;
              },
              [&](int i) { return zc[i]; });
          long long h1, l1;
          ok &= canon::split(p, h1, l1);
          hi += h1;
          lo += l1;
        }
      }
      for (int c = lane + 32 * RT_PRE; c < nsl; c += 32) {   // larger H only
        const float *zc = zt + zpos(c * canon::SLICE);
        const float *wc = reinterpret_cast<const float *>(w4 + c * 4);
        long long h1, l1;
        ok &= canon::split(canon::slice_dot([&](int i) { return __ldg(wc + i); }, [&](int i) { return zc[i]; }), h1,
                           l1);
        hi += h1;
        lo += l1;
      }
      canon::warp_sum_fix(hi, lo);
      if (lane == 0) a.logits[(size_t)t * E + e_row] = canon::logit(canon::join(hi, lo), rinv_s[t], b);
    }
    if (!ok) range_bad = 1;
  }

  // the last CTA to finish selects the experts of every token (one warp each)
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    if (range_bad) set_status(a.status, DEV_RANGE);
    is_last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1u) ? 1u : 0u;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int t = warp; t < T; t += RT_WARPS)
    warp_topk_gates(a.logits + (size_t)t * E, E, a.k, a.idx + t * a.k, a.gate + t * a.k, &topk_sc[warp]);
  __syncthreads();
  if (tid == 0) atomicExch(a.ticket, 0u);
}

// x_out = RMSNorm(x + y), one CTA per token, with the sum of squares of
// decode_canon.cuh (warp 0).
__global__ void __launch_bounds__(256) rmsnorm_residual_kernel(const float *x, const float *y, float eps, float *out,
                                                               int H) {
  __shared__ float inv;
  const int t = blockIdx.x, tid = threadIdx.x;
  const float *xr = x + (size_t)t * H;
  const float *yr = y + (size_t)t * H;
  if (tid < 32) {
    const double ss = canon::warp_sumsq(
        [&](int c) {
          const int b = c * canon::SLICE;
          return canon::slice_sumsq([&](int i) { return __fadd_rn(xr[b + i], yr[b + i]); });
        },
        H / canon::SLICE);
    if (tid == 0) inv = __double2float_rn(canon::norm_rinv(ss, H, eps));
  }
  __syncthreads();
  for (int h = tid; h < H; h += 256) out[(size_t)t * H + h] = __fmul_rn(__fadd_rn(xr[h], yr[h]), inv);
}

size_t decode_ws_bytes(int T, int E) { return (((size_t)T * E * sizeof(double) + 255) & ~(size_t)255) + 256; }

qmoe_status launch_route_decode(const RouteArgs &a, bool resid, cudaStream_t s) {
  const size_t smem = route_smem_bytes(a.T, a.H);
  const void *fn = resid ? (const void *)route_decode_kernel<true> : (const void *)route_decode_kernel<false>;
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return QMOE_ERR_CUDA;
  // static + dynamic shared memory must fit one SM's opt-in limit; above the
  // default 48 KB the kernel's dynamic limit has to be raised
  if (smem + fa.sharedSizeBytes > max_smem_optin()) return QMOE_ERR_UNSUPPORTED;
  if (smem + fa.sharedSizeBytes > 48 * 1024 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMOE_ERR_CUDA;
  const int grid = (a.E + RT_WARPS - 1) / RT_WARPS;
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

// Every call looks the array's address up again (cudaGetSymbolAddress
// allocates nothing): after a device reset, or in another context on the same
// device, the module is loaded afresh and the array may sit elsewhere. The
// first call that sees an address on a device zeroes the array there
// (synchronous; the ticket must start at zero).
qmoe_status fixed_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QMOE_ERR_CUDA;
  if (dev < 0 || dev >= FIXED_MAX_DEVICES) return QMOE_ERR_UNSUPPORTED;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return QMOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_fixed_mutex);
  if (g_fixed_ptr[dev] != p) {
    if (cudaMemset(p, 0, QMOE_ROUTE_FIXED_SCRATCH_BYTES) != cudaSuccess) return QMOE_ERR_CUDA;
    g_fixed_ptr[dev] = p;
  }
  *out = p;
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
  if (H % canon::SLICE) return QMOE_ERR_UNSUPPORTED;
  rmsnorm_residual_kernel<<<T, 256, 0, (cudaStream_t)stream>>>(x_in, y, eps, x_out, H);
  note_launch();
  return cuda_status(cudaGetLastError());
}
