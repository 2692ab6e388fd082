// Router for prefill chunks (more than 8 tokens, or bf16 activations):
// a float64 logit GEMM over register tiles, then one warp per token for the
// top-k selection and the renormalised gates.
//
// Every product x[t,h] * Wr[e,h] (bf16 or fp32 times fp32) is exact in
// float64, and the sums are float64, so the logits match correctly rounded
// values to within about 2^-40 relative; the selection rule is the decode
// router's (value descending, lower expert index on equal values).
#include <cuda_bf16.h>

#include "common.cuh"
#include "route_common.cuh"

namespace qmoe {
namespace {

constexpr int LG_TT = 64;    // tokens per CTA
constexpr int LG_TE = 128;   // experts per CTA
constexpr int LG_KC = 16;    // reduction elements per shared-memory chunk
constexpr int LG_THREADS = 128;

template <int XDT>
__device__ __forceinline__ double load_x(const void *x, size_t i) {
  if (XDT == QMOE_BF16) {
    const unsigned short b = static_cast<const unsigned short *>(x)[i];
    return (double)__uint_as_float((uint32_t)b << 16);
  } else {
    return (double)static_cast<const float *>(x)[i];
  }
}

// logits[t, e] = sum_h x[t,h] * Wr[e,h] + bias[e] for a 64-token x 128-expert
// tile. Thread (ty, tx) owns tokens ty + 8i and experts tx + 16j (i, j < 8).
// Token and expert indices beyond T / E are clamped on load and not stored.
template <int XDT>
__global__ void __launch_bounds__(LG_THREADS, 2) logits_kernel(const void *__restrict__ x,
                                                              const float *__restrict__ Wr,
                                                              const float *__restrict__ bias, int T, int H, int E,
                                                              double *__restrict__ logits) {
  __shared__ double xs[LG_KC][LG_TT];
  __shared__ double ws[LG_KC][LG_TE];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int t0 = blockIdx.x * LG_TT, e0 = blockIdx.y * LG_TE;
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  for (int k0 = 0; k0 < H; k0 += LG_KC) {
    __syncthreads();
#pragma unroll
    for (int m = 0; m < (LG_TT * LG_KC) / LG_THREADS; ++m) {
      const int id = tid + LG_THREADS * m, t = id / LG_KC, kk = id % LG_KC;
      const int tg = min(t0 + t, T - 1);
      xs[kk][t] = load_x<XDT>(x, (size_t)tg * H + k0 + kk);
    }
#pragma unroll
    for (int m = 0; m < (LG_TE * LG_KC) / LG_THREADS; ++m) {
      const int id = tid + LG_THREADS * m, e = id / LG_KC, kk = id % LG_KC;
      const int eg = min(e0 + e, E - 1);
      ws[kk][e] = (double)Wr[(size_t)eg * H + k0 + kk];
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < LG_KC; ++kk) {
      double xv[8], wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) xv[i] = xs[kk][ty + 8 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) wv[j] = ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(xv[i], wv[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = e0 + tx + 16 * j;
    if (e >= E) continue;
    const double b = bias ? (double)bias[e] : 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int t = t0 + ty + 8 * i;
      if (t < T) logits[(size_t)t * E + e] = acc[i][j] + b;
    }
  }
}

constexpr int TK_WARPS = 8;

__global__ void __launch_bounds__(TK_WARPS * 32) topk_kernel(const double *__restrict__ logits, int T, int E, int k,
                                                             int32_t *__restrict__ idx, float *__restrict__ gate) {
  __shared__ TopkScratch sc[TK_WARPS];
  const int warp = threadIdx.x >> 5;
  const int t = blockIdx.x * TK_WARPS + warp;
  if (t >= T) return;
  const double *l = logits + (size_t)t * E;
  warp_topk_gates_get([&](int e) { return __ldg(l + e); }, E, k, idx + (size_t)t * k, gate + (size_t)t * k,
                      &sc[warp]);
}

}  // namespace

size_t route_prefill_ws_bytes(int T, int E) { return (((size_t)T * E * sizeof(double) + 255) & ~(size_t)255) + 256; }

qmoe_status route_prefill(const float *Wr, const float *bias, const void *x, int x_dtype, int T, int H, int E, int k,
                          int32_t *idx, float *gate, void *ws, size_t ws_bytes, int32_t *, cudaStream_t s) {
  if (H % LG_KC) return QMOE_ERR_UNSUPPORTED;
  if (ws_bytes < route_prefill_ws_bytes(T, E)) return QMOE_ERR_WORKSPACE;
  double *logits = static_cast<double *>(ws);
  const dim3 grid((T + LG_TT - 1) / LG_TT, (E + LG_TE - 1) / LG_TE);
  if (x_dtype == QMOE_BF16)
    logits_kernel<QMOE_BF16><<<grid, LG_THREADS, 0, s>>>(x, Wr, bias, T, H, E, logits);
  else
    logits_kernel<QMOE_F32><<<grid, LG_THREADS, 0, s>>>(x, Wr, bias, T, H, E, logits);
  note_launch();
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return cuda_status(err);
  topk_kernel<<<(T + TK_WARPS - 1) / TK_WARPS, TK_WARPS * 32, 0, s>>>(logits, T, E, k, idx, gate);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace qmoe
