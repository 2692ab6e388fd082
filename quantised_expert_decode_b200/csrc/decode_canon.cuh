// Floating-point steps of decoding, written once for every decode path.
//
// The per-layer kernels (router with its residual RMSNorm, expert FFN, final
// norm) and the fused layer-stack kernel split the same work differently
// across threads and CTAs. A token's routes, gates and activations still come
// out bit for bit the same on both paths, and whatever verify batch the token
// sits in, because every rounding step below is fixed here and every sum whose
// parts are formed in different places is an exact integer sum:
//
//   slices     the hidden axis is cut into 16-element slices c (h = 16c + i);
//   partials   a slice's router partial sum_i Wr[e][16c+i] z[16c+i] and its
//              sum of squares sum_i z[16c+i]^2 are float64 fma chains in
//              element order i = 0..15;
//   logits     each router partial is rounded to an integer in units of
//              2^-32 (one rounding, to nearest); integers add exactly in any
//              order, so a row summed by one warp and a row summed over 128
//              CTAs with atomics agree;
//   squares    the slice sums of squares are added in one fixed order: lane l
//              of a warp adds slices l, l + 32, l + 64, ... in turn, then the
//              32 lane sums meet in a butterfly (xor 16, 8, 4, 2, 1); the fused
//              kernel stores the slice sums and every CTA adds them this way;
//   norm       rinv = 1 / sqrt(SS / H + eps) in float64; the activations the
//              experts see are x = z * (float)rinv; router logits are
//              (sum of partials of z) * rinv + bias, using Wr (z / rms) =
//              (Wr z) / rms, so the logits need no second pass after the norm;
//   combine    y = sum_j gate_j * r_j in slot order, one rounding per multiply
//              and per add; z_next = x + y.
//
// A router partial of magnitude 2^19 or more (or NaN) is reported through the
// device status (DEV_RANGE) instead: below it the integer stays under 2^51, so
// one magic-number addition rounds it, and the sum of up to 2^12 slices
// (H <= 65,536) cannot overflow 64 bits. Slice partials of normalised
// activations are of order 1; the rounding (at most 2^-33 a slice) moves a
// 128-slice logit by less than 2e-8.
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace qmoe {
namespace canon {
namespace {

constexpr int SLICE = 16;
constexpr double FIX_UNIT = 4294967296.0;                   // 2^32
constexpr double FIX_UNIT_INV = 1.0 / 4294967296.0;         // 2^-32
constexpr double FIX_RANGE = 524288.0;                       // 2^19
constexpr double MAGIC = 6755399441055744.0;                 // 1.5 * 2^52: its ulp is 1

// p -> v = round(p * 2^32) in one fused multiply-add: p * 2^32 is exact, the
// addition of 1.5 * 2^52 rounds it to an integer (to nearest, ties to even;
// the sum stays in [2^52, 2^53) for |p| < 2^19), and the integer sits in the
// sum's low mantissa bits: v = bits(t) - bits(1.5 * 2^52). No conversion
// instruction. Returns false (and 0) when |p| >= 2^19 or p is NaN.
__device__ __forceinline__ bool fix(double p, long long &v) {
  if (!(fabs(p) < FIX_RANGE)) {
    v = 0;
    return false;
  }
  const double t = __fma_rn(p, FIX_UNIT, MAGIC);
  v = __double_as_longlong(t) - __double_as_longlong(MAGIC);
  return true;
}

// int64 -> float64 without a conversion instruction: each 32-bit half goes
// through the 2^52 magic number (exact), then hi * 2^32 + lo, exact below 2^53
// and rounded once (to nearest) above.
__device__ __forceinline__ double i64_to_f64(long long v) {
  const double h = __dsub_rn(__hiloint2double(0x43300000, (int)(((unsigned long long)v >> 32) ^ 0x80000000u)),
                             4503601774854144.0);          // 2^52 + 2^31
  const double l = __dsub_rn(__hiloint2double(0x43300000, (int)(unsigned)v), 4503599627370496.0);   // 2^52
  return __fma_rn(h, 4294967296.0, l);
}

// An exact integer total -> float64 (one rounding above 2^53, then an exact
// scaling).
__device__ __forceinline__ double unfix(long long v) { return __dmul_rn(i64_to_f64(v), FIX_UNIT_INV); }

// float -> float64, exactly, for normal numbers by moving the bits (IEEE 754
// binary32 -> binary64: the exponent rebiased by 1023 - 127, the 23 mantissa
// bits placed at the top of the 52); zero, subnormals, infinities and NaN go
// through the conversion instruction. Integer operations only on the common
// path: the conversion unit issues at a small fraction of the integer rate and
// was the bottleneck of the router's dot products.
__device__ __forceinline__ double f2d(float f) {
  const unsigned u = __float_as_uint(f);
  const unsigned a = u & 0x7fffffffu;
  if (a - 0x00800000u < 0x7f000000u)
    return __hiloint2double((int)((u & 0x80000000u) | ((a >> 3) + 0x38000000u)), (int)(a << 29));
  return (double)f;
}

// Router partial of one slice: w(i), z(i) for i = 0..15.
template <class W, class Z>
__device__ __forceinline__ double slice_dot(W w, Z z) {
  double p = 0.0;
#pragma unroll
  for (int i = 0; i < SLICE; ++i) p = fma(f2d(w(i)), f2d(z(i)), p);
  return p;
}

// slice_dot with the activations already widened, zd[i] = f2d(z(i)): the same
// value, for loops that reuse one slice of z over many router rows.
template <class W>
__device__ __forceinline__ double slice_dot_wide(W w, const double (&zd)[SLICE]) {
  double p = 0.0;
#pragma unroll
  for (int i = 0; i < SLICE; ++i) p = fma(f2d(w(i)), zd[i], p);
  return p;
}

// Sum of squares of one slice.
template <class Z>
__device__ __forceinline__ double slice_sumsq(Z z) {
  double p = 0.0;
#pragma unroll
  for (int i = 0; i < SLICE; ++i) {
    const double v = f2d(z(i));
    p = fma(v, v, p);
  }
  return p;
}

// Sum of squares of a token from its slice sums q(c), c < nsl, in the fixed
// order above; every lane of the calling warp returns the same value.
// Up to PRE slice sums per lane are fetched before any is added, so slice sums
// read from global memory cost one round trip, not one per slice.
// The same order with the lane's first PRE slice sums v[m] (slice lane + 32 m)
// already formed; slices from 32 PRE on come from q(c).
template <int PRE, class Q>
__device__ __forceinline__ double warp_sum_slices(const double (&v)[PRE], Q q, int nsl) {
  const int lane = threadIdx.x & 31;
  double s = 0.0;
#pragma unroll
  for (int m = 0; m < PRE; ++m)
    if (lane + 32 * m < nsl) s = __dadd_rn(s, v[m]);
  for (int c = lane + 32 * PRE; c < nsl; c += 32) s = __dadd_rn(s, q(c));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
  return s;
}

template <int PRE = 4, class Q>
__device__ __forceinline__ double warp_sumsq(Q q, int nsl) {
  const int lane = threadIdx.x & 31;
  double v[PRE];
#pragma unroll
  for (int m = 0; m < PRE; ++m) v[m] = lane + 32 * m < nsl ? q(lane + 32 * m) : 0.0;
  return warp_sum_slices<PRE>(v, q, nsl);
}

// 1 / rms from the sum of squares of H elements.
__device__ __forceinline__ double norm_rinv(double ss, int H, float eps) {
  return __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)H), (double)eps)));
}

__device__ __forceinline__ double logit(double partial_sum, double rinv, double bias) {
  return __dadd_rn(__dmul_rn(partial_sum, rinv), bias);
}

// One slot of the combine: y + g * r.
__device__ __forceinline__ float combine_step(float y, float g, float r) { return __fadd_rn(y, __fmul_rn(g, r)); }

__device__ __forceinline__ float silu(float a) { return __fdiv_rn(a, __fadd_rn(1.0f, expf(-a))); }

__device__ __forceinline__ float hval(float a_g, float a_u) { return __fmul_rn(silu(a_g), a_u); }



}  // namespace
}  // namespace canon
}  // namespace qmoe
