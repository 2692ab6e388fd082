// Router for prefill chunks (more than 8 tokens, or bf16 activations).
//
// The selection must be the exact one (largest logits, lower expert index on
// equal values) for every token, and the gates need accurate logits of the
// selected experts. Forming all T x E logits in float64 costs as much as the
// expert GEMMs, so the router works in two passes:
//
// 1. Candidates, on the integer tensor cores. Every token row x_t and router
//    row w_e is quantised to 16-bit fixed point (scales s_x = max|x_t| / 32639,
//    s_w = max|w_e| / 32639), split into two signed 8-bit limbs, and the
//    limb products are summed exactly in int32 (mma m16n8k32 s8 x s8). The
//    approximate logit a = s_x s_w sum X W (+ b) differs from the true one by
//    at most B = 0.51 (s_x |w_e|_1 + s_w (|x_t|_1 + 0.51 H s_x)) (each value
//    is within 0.51 of its scale from its quantised value), plus float64
//    rounding slack. With tau the k-th largest a of the token and Bmax its
//    largest bound, every expert of the true top-k has a + B >= tau - Bmax;
//    those experts are the candidates (typically k + 1 or k + 2).
// 2. Exact selection: float64 logits (exact products, float64 sums) of the
//    candidates only, the top-k among them by the selection rule, and the
//    renormalised gates from those logits, as the decode router computes them.
//    A token with more than RQ_CAND candidates (a degenerate router with many
//    near-equal logits) gets float64 logits for all experts instead.
#include <cuda_bf16.h>

#include "common.cuh"
#include "route_common.cuh"

namespace qmoe {
namespace {

constexpr int RQ_TT = 64;            // tokens per GEMM CTA
constexpr int RQ_TE = 64;            // experts per GEMM CTA
constexpr int RQ_KC = 64;            // reduction elements per shared-memory chunk
constexpr int RQ_THREADS = 256;
constexpr int RQ_ROW = RQ_KC + 16;   // padded int8 row: conflict-free fragment loads
constexpr int RQ_XMAX = 32639;       // 127 * 256 + 127: two balanced signed 8-bit limbs
constexpr int RQ_CAND = 64;
constexpr int RQ_SEL_WARPS = 8;

struct Scales {
  float *sx, *sw;          // [T], [E] quantisation scales
  double *n1x, *n1w;       // [T], [E] L1 norms of the rows
};

template <int XDT>
__device__ __forceinline__ float load_xf(const void *x, size_t i) {
  if (XDT == QMOE_BF16) return __uint_as_float((uint32_t) static_cast<const unsigned short *>(x)[i] << 16);
  return static_cast<const float *>(x)[i];
}

// Four consecutive activations of token row x_t as floats (bf16 is exact in fp32).
template <int XDT>
__device__ __forceinline__ float4 load_x4(const void *x, size_t i) {
  if (XDT == QMOE_BF16) {
    const uint2 u = *reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(x) + i);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
  }
  return *reinterpret_cast<const float4 *>(static_cast<const float *>(x) + i);
}

// One warp per row: token rows 0..T-1, then router rows T..T+E-1.
template <int XDT>
__global__ void __launch_bounds__(256) rq_scale_kernel(const void *__restrict__ x, const float *__restrict__ Wr, int T,
                                                       int E, int H, Scales sc) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= T + E) return;
  float amax = 0.0f;
  double n1 = 0.0;
  if (row < T) {
    for (int h = lane; h < H; h += 32) {
      const float v = load_xf<XDT>(x, (size_t)row * H + h);
      amax = fmaxf(amax, fabsf(v));
      n1 += fabs((double)v);
    }
  } else {
    const float *w = Wr + (size_t)(row - T) * H;
    for (int h = lane; h < H; h += 32) {
      const float v = w[h];
      amax = fmaxf(amax, fabsf(v));
      n1 += fabs((double)v);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  n1 = warp_sum_d(n1);
  if (lane == 0) {
    const float s = amax > 0.0f ? amax / (float)RQ_XMAX : 0.0f;
    if (row < T) {
      sc.sx[row] = s;
      sc.n1x[row] = n1;
    } else {
      sc.sw[row - T] = s;
      sc.n1w[row - T] = n1;
    }
  }
}

__device__ __forceinline__ void mma_s8s8(int &d0, int &d1, int &d2, int &d3, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d0), "+r"(d1), "+r"(d2), "+r"(d3)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Quantise v with scale inverse inv into X = 256 hi + lo (|X| <= RQ_XMAX).
__device__ __forceinline__ void quant2(float v, float inv, int &hi, int &lo) {
  const int X = max(-RQ_XMAX, min(RQ_XMAX, __float2int_rn(v * inv)));
  lo = ((X + 128) & 255) - 128;
  hi = (X - lo) >> 8;
}

__device__ __forceinline__ uint32_t pack4b(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
         ((uint32_t)(d & 0xff) << 24);
}

// Approximate logits of a 64-token x 64-expert tile. Shared memory holds the
// hi and lo limb planes of the current K chunk, [row][RQ_ROW] bytes; global
// loads of the next chunk are held in registers while the current one is
// multiplied. Warp (wm, wn) = (w % 4, w / 4) owns tokens 16 wm.. and experts
// 32 wn.. (4 n-tiles of 8); accumulators: hi*hi, hi*lo + lo*hi, lo*lo.
template <int XDT>
__global__ void __launch_bounds__(RQ_THREADS, 2) rq_gemm_kernel(const void *__restrict__ x,
                                                                const float *__restrict__ Wr,
                                                                const float *__restrict__ bias, int T, int E, int H,
                                                                Scales sc, double *__restrict__ approx) {
  __shared__ __align__(16) uint8_t xs[2][RQ_TT * RQ_ROW];      // [plane][row * RQ_ROW]
  __shared__ __align__(16) uint8_t wsm[2][RQ_TE * RQ_ROW];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int t0 = blockIdx.x * RQ_TT, e0 = blockIdx.y * RQ_TE;
  // loader roles: x and w: row tid / 4, 16 values from column (tid % 4) * 16
  const int xr = tid >> 2, xc = (tid & 3) * 16, wr = tid >> 2, wc = (tid & 3) * 16;
  const int xtok = min(t0 + xr, T - 1), wexp = min(e0 + wr, E - 1);
  const float xinv = sc.sx[xtok] > 0.0f ? 1.0f / sc.sx[xtok] : 0.0f;
  const float winv = sc.sw[wexp] > 0.0f ? 1.0f / sc.sw[wexp] : 0.0f;
  float xv[16], wv[16];
  auto gload = [&](int k0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = load_x4<XDT>(x, (size_t)xtok * H + k0 + xc + 4 * q);
      xv[4 * q] = f.x;
      xv[4 * q + 1] = f.y;
      xv[4 * q + 2] = f.z;
      xv[4 * q + 3] = f.w;
    }
    const float4 *wp = reinterpret_cast<const float4 *>(Wr + (size_t)wexp * H + k0 + wc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = __ldg(wp + i);
      wv[4 * i] = f.x;
      wv[4 * i + 1] = f.y;
      wv[4 * i + 2] = f.z;
      wv[4 * i + 3] = f.w;
    }
  };
  auto sstore = [&]() {
    int h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int i = 0; i < 4; ++i) quant2(xv[4 * q + i], xinv, h[i], l[i]);
      *reinterpret_cast<uint32_t *>(&xs[0][xr * RQ_ROW + xc + 4 * q]) = pack4b(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint32_t *>(&xs[1][xr * RQ_ROW + xc + 4 * q]) = pack4b(l[0], l[1], l[2], l[3]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int i = 0; i < 4; ++i) quant2(wv[4 * q + i], winv, h[i], l[i]);
      *reinterpret_cast<uint32_t *>(&wsm[0][wr * RQ_ROW + wc + 4 * q]) = pack4b(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<uint32_t *>(&wsm[1][wr * RQ_ROW + wc + 4 * q]) = pack4b(l[0], l[1], l[2], l[3]);
    }
  };
  const int wm = warp & 3, wn = warp >> 2;
  int hh[4][4], mid[4][4], ll[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) hh[n][i] = mid[n][i] = ll[n][i] = 0;

  gload(0);
  for (int k0 = 0; k0 < H; k0 += RQ_KC) {
    __syncthreads();   // previous chunk's fragments are read
    sstore();
    __syncthreads();
    if (k0 + RQ_KC < H) gload(k0 + RQ_KC);
#pragma unroll
    for (int ks = 0; ks < RQ_KC; ks += 32) {
      uint32_t ah[4], al[4];
      const int ra = (16 * wm + g) * RQ_ROW + ks + 4 * t4, rb = ra + 8 * RQ_ROW;
      ah[0] = *reinterpret_cast<const uint32_t *>(&xs[0][ra]);
      ah[1] = *reinterpret_cast<const uint32_t *>(&xs[0][rb]);
      ah[2] = *reinterpret_cast<const uint32_t *>(&xs[0][ra + 16]);
      ah[3] = *reinterpret_cast<const uint32_t *>(&xs[0][rb + 16]);
      al[0] = *reinterpret_cast<const uint32_t *>(&xs[1][ra]);
      al[1] = *reinterpret_cast<const uint32_t *>(&xs[1][rb]);
      al[2] = *reinterpret_cast<const uint32_t *>(&xs[1][ra + 16]);
      al[3] = *reinterpret_cast<const uint32_t *>(&xs[1][rb + 16]);
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const int rw = (32 * wn + 8 * n + g) * RQ_ROW + ks + 4 * t4;
        const uint32_t bh0 = *reinterpret_cast<const uint32_t *>(&wsm[0][rw]);
        const uint32_t bh1 = *reinterpret_cast<const uint32_t *>(&wsm[0][rw + 16]);
        const uint32_t bl0 = *reinterpret_cast<const uint32_t *>(&wsm[1][rw]);
        const uint32_t bl1 = *reinterpret_cast<const uint32_t *>(&wsm[1][rw + 16]);
        mma_s8s8(hh[n][0], hh[n][1], hh[n][2], hh[n][3], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
        mma_s8s8(mid[n][0], mid[n][1], mid[n][2], mid[n][3], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
        mma_s8s8(mid[n][0], mid[n][1], mid[n][2], mid[n][3], al[0], al[1], al[2], al[3], bh0, bh1);
        mma_s8s8(ll[n][0], ll[n][1], ll[n][2], ll[n][3], al[0], al[1], al[2], al[3], bl0, bl1);
      }
    }
  }
  // accumulator (row, col) of fragment i: rows g / g+8, columns 2 t4 + (i & 1)
#pragma unroll
  for (int n = 0; n < 4; ++n) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = t0 + 16 * wm + g + (i >> 1) * 8;
      const int e = e0 + 32 * wn + 8 * n + 2 * t4 + (i & 1);
      if (tok < T && e < E) {
        const long long q = 65536LL * hh[n][i] + 256LL * mid[n][i] + (long long)ll[n][i];
        double v = (double)q * ((double)sc.sx[tok] * (double)sc.sw[e]);
        if (bias) v += (double)bias[e];
        approx[(size_t)tok * E + e] = v;
      }
    }
  }
}

// Bound on |approx - exact logit| for one (token, expert) pair.
__device__ __forceinline__ double rq_bound(float sx, double n1x, float sw, double n1w, int H, double a) {
  const double b = 0.51 * ((double)sx * n1w + (double)sw * (n1x + 0.51 * (double)H * (double)sx));
  return b * (1.0 + 1e-9) + 1e-12 * (fabs(a) + 1.0);
}

// Exact-product float64 logits of token t for experts e0 and e1 (one warp;
// e1 < 0: only e0). Lane l takes elements 4l..4l+3 of every 128-element chunk.
template <int XDT>
__device__ __forceinline__ void exact_logits2(const void *x, const float *Wr, const float *bias, int t, int e0, int e1,
                                              int H, int lane, double &out0, double &out1) {
  double p0 = 0.0, p1 = 0.0;
  const float *w0 = Wr + (size_t)e0 * H, *w1 = Wr + (size_t)(e1 >= 0 ? e1 : e0) * H;
#pragma unroll 4
  for (int h = 4 * lane; h < H; h += 128) {
    const float4 xv = load_x4<XDT>(x, (size_t)t * H + h);
    const float4 a = __ldg(reinterpret_cast<const float4 *>(w0 + h));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(w1 + h));
    p0 = fma((double)xv.x, (double)a.x, p0);
    p0 = fma((double)xv.y, (double)a.y, p0);
    p0 = fma((double)xv.z, (double)a.z, p0);
    p0 = fma((double)xv.w, (double)a.w, p0);
    p1 = fma((double)xv.x, (double)b.x, p1);
    p1 = fma((double)xv.y, (double)b.y, p1);
    p1 = fma((double)xv.z, (double)b.z, p1);
    p1 = fma((double)xv.w, (double)b.w, p1);
  }
  p0 = warp_sum_d(p0);
  p1 = warp_sum_d(p1);
  out0 = bias ? p0 + (double)bias[e0] : p0;
  out1 = (e1 >= 0 && bias) ? p1 + (double)bias[e1] : p1;
}

struct SelScratch {
  int cand[RQ_CAND];
  double cand_v[RQ_CAND];
  int sel_e[TOPK_MAX_K];
  double sel_v[TOPK_MAX_K];
  TopkScratch tks;
};

// One warp per token; M = ceil(E / 32) values per lane.
template <int M, int XDT>
__device__ void rq_select_token(const void *x, const float *Wr, const float *bias, int t, int E, int H, int k,
                                Scales sc, double *approx_row, int32_t *idx, float *gate, SelScratch *s) {
  const int lane = threadIdx.x & 31;
  const float sx = sc.sx[t];
  const double n1x = sc.n1x[t];
  double v[M], bnd[M];
  double bmax = 0.0;
#pragma unroll
  for (int i = 0; i < M; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? approx_row[e] : -INFINITY;
    bnd[i] = e < E ? rq_bound(sx, n1x, sc.sw[e], sc.n1w[e], H, v[i]) : 0.0;
    bmax = fmax(bmax, bnd[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bmax = fmax(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
  // tau: the k-th largest approximate logit (k rounds removing one maximum each)
  unsigned taken = 0;
  double tau = -INFINITY;
  for (int r = 0; r < k; ++r) {
    double m = -INFINITY;
    int mi = -1;
#pragma unroll
    for (int i = 0; i < M; ++i)
      if (!((taken >> i) & 1u) && v[i] > m) {
        m = v[i];
        mi = i;
      }
    double wm = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wm = fmax(wm, __shfl_xor_sync(0xffffffffu, wm, o));
    const unsigned owners = __ballot_sync(0xffffffffu, mi >= 0 && m == wm);
    if (owners && lane == __ffs(owners) - 1) taken |= 1u << mi;
    tau = wm;
  }
  const double lowk = tau - bmax;
  // candidates: every expert whose approximate logit plus its bound reaches lowk
  int mine = 0;
#pragma unroll
  for (int i = 0; i < M; ++i) mine += (lane + 32 * i < E && v[i] + bnd[i] >= lowk) ? 1 : 0;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total > RQ_CAND) {
    // degenerate: float64 logits of every expert, then the general selection
    for (int e = 0; e < E; e += 2) {
      double p0, p1;
      exact_logits2<XDT>(x, Wr, bias, t, e, e + 1 < E ? e + 1 : -1, H, lane, p0, p1);
      if (lane == 0) {
        approx_row[e] = p0;
        if (e + 1 < E) approx_row[e + 1] = p1;
      }
    }
    __syncwarp();
    __threadfence_block();
    warp_topk_gates_get([&](int e) { return approx_row[e]; }, E, k, idx, gate, &s->tks);
    return;
  }
  {
    int pos = incl - mine;
#pragma unroll
    for (int i = 0; i < M; ++i)
      if (lane + 32 * i < E && v[i] + bnd[i] >= lowk) s->cand[pos++] = lane + 32 * i;
  }
  __syncwarp();
  for (int c = 0; c < total; c += 2) {
    double p0, p1;
    exact_logits2<XDT>(x, Wr, bias, t, s->cand[c], c + 1 < total ? s->cand[c + 1] : -1, H, lane, p0, p1);
    if (lane == 0) {
      s->cand_v[c] = p0;
      if (c + 1 < total) s->cand_v[c + 1] = p1;
    }
  }
  __syncwarp();
  // rank the candidates exactly (value descending, lower expert first on ties)
  for (int c = lane; c < total; c += 32) {
    const int e = s->cand[c];
    const double val = s->cand_v[c];
    int rank = 0;
    for (int c2 = 0; c2 < total; ++c2) rank += ranks_above(s->cand_v[c2], s->cand[c2], val, e) ? 1 : 0;
    if (rank < k) {
      s->sel_e[rank] = e;
      s->sel_v[rank] = val;
    }
  }
  __syncwarp();
  float ex = 0.0f;
  if (lane < k) ex = expf((float)(s->sel_v[lane] - s->sel_v[0]));
  const float sum = warp_sum(ex);
  if (lane < k) {
    idx[lane] = s->sel_e[lane];
    gate[lane] = ex / sum;
  }
}

template <int XDT>
__global__ void __launch_bounds__(RQ_SEL_WARPS * 32) rq_select_kernel(const void *__restrict__ x,
                                                                      const float *__restrict__ Wr,
                                                                      const float *__restrict__ bias, int T, int E,
                                                                      int H, int k, Scales sc, double *approx,
                                                                      int32_t *idx, float *gate) {
  __shared__ SelScratch sel[RQ_SEL_WARPS];
  const int warp = threadIdx.x >> 5;
  const int t = blockIdx.x * RQ_SEL_WARPS + warp;
  if (t >= T) return;
  double *row = approx + (size_t)t * E;
  int32_t *it = idx + (size_t)t * k;
  float *gt = gate + (size_t)t * k;
  SelScratch *s = &sel[warp];
  if (E <= 32) rq_select_token<1, XDT>(x, Wr, bias, t, E, H, k, sc, row, it, gt, s);
  else if (E <= 64) rq_select_token<2, XDT>(x, Wr, bias, t, E, H, k, sc, row, it, gt, s);
  else if (E <= 128) rq_select_token<4, XDT>(x, Wr, bias, t, E, H, k, sc, row, it, gt, s);
  else if (E <= 256) rq_select_token<8, XDT>(x, Wr, bias, t, E, H, k, sc, row, it, gt, s);
  else if (E <= 512) rq_select_token<16, XDT>(x, Wr, bias, t, E, H, k, sc, row, it, gt, s);
  else rq_select_token<32, XDT>(x, Wr, bias, t, E, H, k, sc, row, it, gt, s);
}

inline size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

template <int XDT>
qmoe_status rq_launch(const float *Wr, const float *bias, const void *x, int T, int H, int E, int k, int32_t *idx,
                      float *gate, void *ws, cudaStream_t s) {
  char *p = static_cast<char *>(ws);
  double *approx = reinterpret_cast<double *>(p);
  p += up256((size_t)T * E * sizeof(double));
  Scales sc;
  sc.n1x = reinterpret_cast<double *>(p); p += up256((size_t)T * 8);
  sc.n1w = reinterpret_cast<double *>(p); p += up256((size_t)E * 8);
  sc.sx = reinterpret_cast<float *>(p); p += up256((size_t)T * 4);
  sc.sw = reinterpret_cast<float *>(p);
  rq_scale_kernel<XDT><<<(T + E + 7) / 8, 256, 0, s>>>(x, Wr, T, E, H, sc);
  note_launch();
  rq_gemm_kernel<XDT><<<dim3((T + RQ_TT - 1) / RQ_TT, (E + RQ_TE - 1) / RQ_TE), RQ_THREADS, 0, s>>>(x, Wr, bias, T, E,
                                                                                                     H, sc, approx);
  note_launch();
  rq_select_kernel<XDT><<<(T + RQ_SEL_WARPS - 1) / RQ_SEL_WARPS, RQ_SEL_WARPS * 32, 0, s>>>(x, Wr, bias, T, E, H, k,
                                                                                              sc, approx, idx, gate);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace

size_t route_prefill_ws_bytes(int T, int E) {
  return up256((size_t)T * E * sizeof(double)) + up256((size_t)T * 8) + up256((size_t)E * 8) + up256((size_t)T * 4) +
         up256((size_t)E * 4) + 256;
}

qmoe_status route_prefill(const float *Wr, const float *bias, const void *x, int x_dtype, int T, int H, int E, int k,
                          int32_t *idx, float *gate, void *ws, size_t ws_bytes, int32_t *, cudaStream_t s) {
  if (H % RQ_KC || H > 32768) return QMOE_ERR_UNSUPPORTED;
  if (ws_bytes < route_prefill_ws_bytes(T, E)) return QMOE_ERR_WORKSPACE;
  if (x_dtype == QMOE_BF16) return rq_launch<QMOE_BF16>(Wr, bias, x, T, H, E, k, idx, gate, ws, s);
  return rq_launch<QMOE_F32>(Wr, bias, x, T, H, E, k, idx, gate, ws, s);
}

}  // namespace qmoe
