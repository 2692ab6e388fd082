// Router for decode batches (T <= 8): float64 router logits from exact
// fixed-point sums of 16-element slice partials, top-k with ties to the lower
// expert index, renormalised gates; optionally preceded by the residual
// RMSNorm of the previous layer's output. The arithmetic is the one of
// decode_canon.cuh, shared with the fused layer-stack kernel.
//
// Work split. CTA (g, s) owns the 32 experts 32g .. 32g+31 (one per lane) and
// the s-th of ns ranges of 16-element slices of the hidden axis; its warps
// take the range's slices in turn. A lane streams its expert's weights of a
// slice into registers and forms the slice partial of every token at once:
// the activations of the range sit in shared memory as float64 [h][token], so
// one broadcast load serves the whole warp. The slice partials are split into
// exact integers (decode_canon.cuh), summed over the CTA's warps and added
// into the workspace with integer atomics; integer sums do not depend on the
// order, so the logits are the same for any split. The CTA that finishes last
// forms the logits (partial sum / rms + bias), selects every token's experts
// (one warp per token, from shared memory) and clears the sums for the next
// call.
#include <mutex>

#include "common.cuh"
#include "decode_canon.cuh"
#include "route_common.cuh"

namespace qmoe {
namespace {

constexpr int RT_WARPS = 8;
constexpr int RT_THREADS = 32 * RT_WARPS;
constexpr int RT_MAXT = 8;
constexpr int RT_GROUP = 32;               // experts per CTA, one per lane
constexpr int RT_CHUNK = 16;               // slices staged in shared memory at a time
constexpr int RT_PRE = 2;                  // slices per warp whose weights are fetched before the wait
static_assert(RT_CHUNK * 16 == 32 * RT_WARPS, "a whole chunk is one element per thread and token");

struct RouteArgs {
  const float *Wr;
  const float *bias;
  const float *x;
  const float *y;      // residual input (RESID only)
  float *x_out;        // normalised activations (RESID only)
  float eps;
  int T, H, E, k;
  int ns;              // hidden-axis ranges per expert group
  int32_t *idx;
  float *gate;
  unsigned long long *lacc;   // workspace [T][E] exact partial-logit sums (2^-32 units, two's complement)
  unsigned *ticket;           // workspace
  int32_t *status;
};

// Dynamic shared memory of one CTA: the largest of the staged activations
// (float64 [RT_CHUNK * 16][TT]), the per-warp integer sums
// ([RT_WARPS][TT][32]) and, in the last CTA, the logits ([T][E]).
inline size_t route_smem_bytes(int TT, int E) {
  size_t z = (size_t)RT_CHUNK * canon::SLICE * TT * 8;
  size_t r = (size_t)RT_WARPS * TT * RT_GROUP * 8;
  size_t l = (size_t)TT * E * 8;
  size_t m = z > r ? z : r;
  return m > l ? m : l;
}

// One warp: token t's 1 / rms from z = x + y (decode_canon.cuh's order) and
// x_out[t] = z * (float)(1 / rms). Up to H = 2048 a lane keeps its four
// slices of z in registers, so x and y are read once, all loads in flight.
__device__ __forceinline__ float4 add4(float4 u, float4 v) {
  return make_float4(__fadd_rn(u.x, v.x), __fadd_rn(u.y, v.y), __fadd_rn(u.z, v.z), __fadd_rn(u.w, v.w));
}
__device__ __forceinline__ float4 scale4(float4 u, float s) {
  return make_float4(__fmul_rn(u.x, s), __fmul_rn(u.y, s), __fmul_rn(u.z, s), __fmul_rn(u.w, s));
}
__device__ __forceinline__ float comp4(const float4 &u, int i) { return i == 0 ? u.x : i == 1 ? u.y : i == 2 ? u.z : u.w; }

__device__ double resid_norm_token(const RouteArgs &a, int t) {
  const int lane = threadIdx.x & 31, H = a.H, nsl = H / canon::SLICE;
  const float4 *x4 = reinterpret_cast<const float4 *>(a.x + (size_t)t * H);
  const float4 *y4 = reinterpret_cast<const float4 *>(a.y + (size_t)t * H);
  float4 *o4 = reinterpret_cast<float4 *>(a.x_out + (size_t)t * H);
  auto zslice = [&](int c) {
    return canon::slice_sumsq([&](int i) {
      return __fadd_rn(__ldcg(a.x + (size_t)t * H + c * canon::SLICE + i), __ldcg(a.y + (size_t)t * H + c * canon::SLICE + i));
    });
  };
  if (nsl <= 128) {
    float4 z[4][4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int c = lane + 32 * m;
#pragma unroll
      for (int q = 0; q < 4; ++q) z[m][q] = c < nsl ? add4(__ldcg(x4 + 4 * c + q), __ldcg(y4 + 4 * c + q))
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    double v[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) v[m] = canon::slice_sumsq([&](int i) { return comp4(z[m][i >> 2], i & 3); });
    const double r = canon::norm_rinv(canon::warp_sum_slices<4>(v, zslice, nsl), H, a.eps);
    const float inv = __double2float_rn(r);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int c = lane + 32 * m;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (c < nsl) o4[4 * c + q] = scale4(z[m][q], inv);
    }
    return r;
  }
  const double r = canon::norm_rinv(canon::warp_sumsq(zslice, nsl), H, a.eps);
  const float inv = __double2float_rn(r);
  for (int h4 = lane; h4 < H / 4; h4 += 32) o4[h4] = scale4(add4(__ldcg(x4 + h4), __ldcg(y4 + h4)), inv);
  return r;
}

// One warp: token t's logits from the exact sums (lane l: experts l + 32 j),
// written to lg (shared memory) for the candidates' values, keys kept in
// registers; the sums are cleared for the next call; then the selection.
template <int M>
__device__ __forceinline__ void route_token_select(const RouteArgs &a, int t, double rinv, double *lg,
                                                   TopkScratch *sc) {
  const int lane = threadIdx.x & 31, E = a.E;
  unsigned long long *ph = a.lacc + (size_t)t * E;
  unsigned long long hv[M];
  float bv[M];
#pragma unroll
  for (int j = 0; j < M; ++j) {
    const int e = lane + 32 * j;
    hv[j] = 0ull;
    bv[j] = 0.0f;
    if (e < E) {
      hv[j] = __ldcg(ph + e);
      if (a.bias) bv[j] = __ldg(a.bias + e);
    }
  }
  unsigned key[M];
#pragma unroll
  for (int j = 0; j < M; ++j) {
    const int e = lane + 32 * j;
    key[j] = 0u;
    if (e < E) {
      const double v = canon::logit(canon::unfix((long long)hv[j]), rinv, a.bias ? canon::f2d(bv[j]) : 0.0);
      lg[e] = v;
      key[j] = logit_key(v);
      ph[e] = 0ull;
    }
  }
  __syncwarp();
  warp_topk_keys<M, true>(key, [&](int e) { return lg[e]; }, E, a.k, a.idx + t * a.k, a.gate + t * a.k, sc);
}

template <int TT, bool RESID>
__global__ void __launch_bounds__(RT_THREADS, 1) route_decode_kernel(RouteArgs a) {
  extern __shared__ __align__(16) double rsm[];
  __shared__ unsigned is_last;
  __shared__ int range_bad;
  __shared__ TopkScratch topk_sc[RT_WARPS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.T, H = a.H, E = a.E, nsl = H / canon::SLICE;
  const int g = blockIdx.x / a.ns, sp = blockIdx.x % a.ns;
  const int e = g * RT_GROUP + lane;
  const bool live = e < E;
  const int c0 = (int)((long long)sp * nsl / a.ns), c1 = (int)((long long)(sp + 1) * nsl / a.ns);
  const float4 *wrow = reinterpret_cast<const float4 *>(a.Wr + (size_t)(live ? e : 0) * H);

  // The first slices' weights do not depend on the previous kernel: fetch
  // them before waiting for it.
  float4 wpre[RT_PRE][4];
#pragma unroll
  for (int m = 0; m < RT_PRE; ++m) {
    const int c = c0 + warp + RT_WARPS * m;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      wpre[m][q] = (live && c < c1 && c < c0 + RT_CHUNK) ? __ldg(wrow + c * 4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (tid == 0) range_bad = 0;
  pdl_wait();
  pdl_launch_dependents();

  long long acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0;
  bool ok = true;
  double *zd = rsm;   // [RT_CHUNK * 16][TT]
  int cc = c0;
  // slice c of the staged chunk: every token's partial, split and summed
  auto slice = [&](int c, const float4 (&w4)[4]) {
    double p[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) p[t] = 0.0;
    const double *zc = zd + (size_t)(c - cc) * canon::SLICE * TT;
#pragma unroll
    for (int i = 0; i < canon::SLICE; ++i) {
      const float4 v = w4[i >> 2];
      const double w = canon::f2d((i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w);
      if (TT == 1) {
        p[0] = fma(w, zc[i], p[0]);
      } else {
#pragma unroll
        for (int t = 0; t < TT; t += 2) {
          const double2 z2 = *reinterpret_cast<const double2 *>(zc + i * TT + t);
          p[t] = fma(w, z2.x, p[t]);
          p[t + 1] = fma(w, z2.y, p[t + 1]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      long long v1;
      ok &= canon::fix(p[t], v1);
      acc[t] += v1;
    }
  };
  for (; cc < c1; cc += RT_CHUNK) {
    const int ncs = min(RT_CHUNK, c1 - cc), nh = ncs * canon::SLICE, h0 = cc * canon::SLICE;
    __syncthreads();   // the previous chunk is no longer read
    if (nh == RT_THREADS) {
      // a whole chunk: element h0 + tid of every token, all loads in flight at once
      float xv[TT], yv[TT];
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        xv[t] = yv[t] = 0.0f;
        if (t < T) {
          xv[t] = __ldcg(a.x + (size_t)t * H + h0 + tid);
          if (RESID) yv[t] = __ldcg(a.y + (size_t)t * H + h0 + tid);
        }
      }
#pragma unroll
      for (int t = 0; t < TT; ++t) zd[tid * TT + t] = canon::f2d(RESID ? __fadd_rn(xv[t], yv[t]) : xv[t]);
    } else {
      for (int i = tid; i < TT * nh; i += RT_THREADS) {
        const int t = i / nh, hh = i % nh;
        float z = 0.0f;
        if (t < T) {
          z = __ldcg(a.x + (size_t)t * H + h0 + hh);
          if (RESID) z = __fadd_rn(z, __ldcg(a.y + (size_t)t * H + h0 + hh));
        }
        zd[hh * TT + t] = canon::f2d(z);
      }
    }
    __syncthreads();
    if (cc == c0) {
      if (warp < ncs) slice(cc + warp, wpre[0]);
      if (warp + RT_WARPS < ncs) slice(cc + warp + RT_WARPS, wpre[1]);
    }
    for (int m = cc == c0 ? RT_PRE : 0; warp + RT_WARPS * m < ncs; ++m) {
      const int c = cc + warp + RT_WARPS * m;
      float4 w4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) w4[q] = live ? __ldg(wrow + c * 4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      slice(c, w4);
    }
  }
  if (!ok && live) range_bad = 1;

  // sum the warps' integers, then one pair of atomics per (token, expert)
  __syncthreads();
  unsigned long long *red = reinterpret_cast<unsigned long long *>(rsm);   // [warp][TT][32]
#pragma unroll
  for (int t = 0; t < TT; ++t) red[(warp * TT + t) * RT_GROUP + lane] = (unsigned long long)acc[t];
  __syncthreads();
  for (int i = tid; i < TT * RT_GROUP; i += RT_THREADS) {
    const int t = i / RT_GROUP, ln = i % RT_GROUP;
    const int ee = g * RT_GROUP + ln;
    if (t < T && ee < E) {
      unsigned long long v = 0;
#pragma unroll
      for (int w = 0; w < RT_WARPS; ++w) v += red[(w * TT + t) * RT_GROUP + ln];
      atomicAdd(a.lacc + (size_t)t * E + ee, v);
    }
  }

  // the last CTA to finish selects the experts of every token
  __syncthreads();
  if (tid == 0) {
    if (range_bad) set_status(a.status, DEV_RANGE);
    __threadfence();
    is_last = (atomicAdd(a.ticket, 1u) == gridDim.x - 1u) ? 1u : 0u;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // one warp per token: 1 / rms (RESID), the logits from the exact sums (which
  // are cleared for the next call), the selection
  double *lg = rsm;   // [T][E]
  for (int t = warp; t < T; t += RT_WARPS) {
    const double rinv = RESID ? resid_norm_token(a, t) : 1.0;
    double *lt = lg + (size_t)t * E;
    switch (topk_m(E)) {
      case 4: route_token_select<4>(a, t, rinv, lt, &topk_sc[warp]); break;
      case 8: route_token_select<8>(a, t, rinv, lt, &topk_sc[warp]); break;
      case 16: route_token_select<16>(a, t, rinv, lt, &topk_sc[warp]); break;
      default: route_token_select<32>(a, t, rinv, lt, &topk_sc[warp]); break;
    }
  }
  __syncthreads();
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

// Workspace: the exact sums [T][E] int64, then a 256-byte ticket block.
size_t decode_lacc_bytes(int T, int E) { return (((size_t)T * E * sizeof(unsigned long long)) + 255) & ~(size_t)255; }
size_t decode_ws_bytes(int T, int E) { return decode_lacc_bytes(T, E) + 256; }

template <int TT>
qmoe_status launch_route_tt(RouteArgs a, bool resid, cudaStream_t s) {
  const void *fn = resid ? (const void *)route_decode_kernel<TT, true> : (const void *)route_decode_kernel<TT, false>;
  const size_t smem = route_smem_bytes(TT, a.E);
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return QMOE_ERR_CUDA;
  // static + dynamic shared memory must fit one SM's opt-in limit; above the
  // default 48 KB the kernel's dynamic limit has to be raised
  if (smem + fa.sharedSizeBytes > max_smem_optin()) return QMOE_ERR_UNSUPPORTED;
  if (smem + fa.sharedSizeBytes > 48 * 1024 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMOE_ERR_CUDA;
  // the largest shared-memory carve-out, as the FFN kernels around it use:
  // an SM then need not be reconfigured between the two kernels
  if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return QMOE_ERR_CUDA;
  const int ng = (a.E + RT_GROUP - 1) / RT_GROUP, nsl = a.H / canon::SLICE;
  int ns = num_sms() / ng;
  if (ns > nsl / 8) ns = nsl / 8;
  if (ns < 1) ns = 1;
  a.ns = ns;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(ng * ns));
  cfg.blockDim = dim3(RT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = resid ? cudaLaunchKernelEx(&cfg, route_decode_kernel<TT, true>, a)
                        : cudaLaunchKernelEx(&cfg, route_decode_kernel<TT, false>, a);
  note_launch();
  return cuda_status(e);
}

qmoe_status launch_route_decode(const RouteArgs &a, bool resid, cudaStream_t s) {
  if (a.T <= 1) return launch_route_tt<1>(a, resid, s);
  if (a.T <= 2) return launch_route_tt<2>(a, resid, s);
  if (a.T <= 4) return launch_route_tt<4>(a, resid, s);
  return launch_route_tt<8>(a, resid, s);
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
  if (H % 128 || H > 65536) return QMOE_ERR_UNSUPPORTED;   // exact sums of at most 4096 slices
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
  a.lacc = static_cast<unsigned long long *>(workspace);
  a.ticket = reinterpret_cast<unsigned *>(static_cast<char *>(workspace) + decode_lacc_bytes(T, E));
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
  a.lacc = static_cast<unsigned long long *>(workspace);
  a.ticket = reinterpret_cast<unsigned *>(static_cast<char *>(workspace) + decode_lacc_bytes(T, E));
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

constexpr size_t FIXED_SUMS_BYTES = (size_t)QMOE_ROUTE_FIXED_MAX_T * QMOE_ROUTE_FIXED_MAX_E * 8;
static_assert(QMOE_ROUTE_FIXED_SCRATCH_BYTES == FIXED_SUMS_BYTES + 256, "fixed scratch layout");

// [0, FIXED_SUMS_BYTES): the exact partial-logit sums ([T][E] int64, laid
// out for the call's own T and E); then the 256-byte ticket block. Both must
// start at zero, and each completed call leaves them at zero.
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
  if (H % 128 || H > 65536 || k > 16 || k > E) return QMOE_ERR_UNSUPPORTED;
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
  a.lacc = static_cast<unsigned long long *>(scratch);
  a.ticket = reinterpret_cast<unsigned *>(static_cast<char *>(scratch) + FIXED_SUMS_BYTES);
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
