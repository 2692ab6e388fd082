// Decode tile primitives shared by the per-layer FFN kernel and the fused
// layer-stack kernel: activation quantisation into int8 limbs and the integer
// tensor-core dot product of one packed 16-row weight tile.
//
// Contraction: activations of every 32-element block are quantised to 24-bit
// fixed point with a per-block fp32 scale s (X = rint(v / s), |X| <= 8355711)
// and split into three signed 8-bit limbs X = 65536*l2 + 256*l1 + l0. The
// integer MMA m16n8k32 (u8 codes x s8 limbs, s32 accumulate) gives the exact
// sums Q_i = sum q*l_i per block; the block's contribution is
// d * s * (65536*Q2 + 256*Q1 + Q0) + m * s * sum(X). A (token, block) pair
// occupies four MMA columns (l2, l1, 0, l0): lane 2P reads (l2, l1) and lane
// 2P+1 reads (0, l0), so each lane finishes its share in fp32 on its own and
// two pairs share one accumulator tile.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "layout.cuh"

namespace qmoe {
namespace tile {
namespace {  // internal linkage: each translation unit keeps its own copy

constexpr float QMAX = 8355711.0f;         // 127*65536 + 127*256 + 127: three int8 limbs
constexpr int LIMB_REC = 96;               // bytes per (vector, block): l2 | l1 | l0

// Exact int -> float for |v| < 2^22: add into the mantissa of 1.5 * 2^23 and
// subtract it again (two full-rate operations instead of a conversion).
__device__ __forceinline__ float i2f_small(int v) {
  return __int_as_float(0x4B400000 + v) - 12582912.0f;
}

// hi * 256 + lo as a float, exactly, for |hi|, |lo| < 2^16 (the block sums of
// one limb pair: at most 32 * 15 * 128 in magnitude): both convert exactly,
// hi * 256 is exact and the sum stays below 2^24. Four full-rate operations
// and one fused multiply-add, no conversion-unit instruction (those issue at a
// fraction of the rate and were the busiest pipe of the tile loop).
__device__ __forceinline__ float limb_pair(int hi, int lo) { return fmaf(i2f_small(hi), 256.0f, i2f_small(lo)); }

// The same value for a tile of BITS-bit codes. With 2-bit codes each block sum
// is at most 32 * 3 * 128 = 12,288 in magnitude, so hi * 256 + lo stays below
// 2^22 and forms exactly in integers, then converts through the magic number
// in one step (three operations instead of five).
template <int BITS>
__device__ __forceinline__ float limb_pair_b(int hi, int lo) {
  if (BITS == 2) return i2f_small(hi * 256 + lo);
  return limb_pair(hi, lo);
}

__device__ __forceinline__ float h2f(uint32_t bits16) { return __half2float(__ushort_as_half((unsigned short)bits16)); }

// Quantise a 128-element chunk (4 blocks of 32) held one float4 per lane: lane
// j carries elements 4j..4j+3, i.e. block j/8. Writes the three int8 limbs of
// the four blocks and (s, s * sum X) per block. The block's min term uses the
// same quantised values as its code term, so the whole block sees one
// consistent activation s*X and the only error is that of quantising v.
__device__ __forceinline__ int quant_one(float v, float inv) {
  const int X = __float2int_rn(__fmul_rn(v, inv));
  return max(-8355711, min(8355711, X));
}

// Scale of a 32-element block from its largest magnitude a: s = a / QMAX taken
// as a * (1 / QMAX), and the reciprocal used to quantise. Every decode path
// quantises with these two values, so a block's limbs and (s, s * sum X) are
// the same bits wherever it is quantised.
__device__ __forceinline__ void block_scale(float a, float &s, float &inv) {
  s = 0.0f;
  inv = 0.0f;
  if (a > 0.0f) {
    s = __fmul_rn(a, 1.0f / QMAX);
    inv = __frcp_rn(s);
  }
}

// balanced base-256 digits of |X| <= 8355711, each in [-128, 127]
__device__ __forceinline__ void limbs3(int X, int &l2, int &l1, int &l0) {
  l0 = ((X + 128) & 255) - 128;
  const int X1 = (X - l0) >> 8;
  l1 = ((X1 + 128) & 255) - 128;
  l2 = (X1 - l1) >> 8;
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
         ((uint32_t)(d & 0xff) << 24);
}

__device__ __noinline__ void quant_chunk(float4 v, uint8_t *limbs_vec, float2 *lsc_vec, int chunk, int lane) {
  float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
  float s, inv;
  block_scale(a, s, inv);
  const int X0 = quant_one(v.x, inv), X1 = quant_one(v.y, inv), X2 = quant_one(v.z, inv), X3 = quant_one(v.w, inv);
  int a2, a1, a0, b2, b1, b0, c2, c1, c0, d2, d1, d0;
  limbs3(X0, a2, a1, a0);
  limbs3(X1, b2, b1, b0);
  limbs3(X2, c2, c1, c0);
  limbs3(X3, d2, d1, d0);
  const int blk = chunk * 4 + (lane >> 3);
  uint8_t *rec = limbs_vec + (size_t)blk * LIMB_REC + (lane & 7) * 4;
  *reinterpret_cast<uint32_t *>(rec) = pack4(a2, b2, c2, d2);
  *reinterpret_cast<uint32_t *>(rec + 32) = pack4(a1, b1, c1, d1);
  *reinterpret_cast<uint32_t *>(rec + 64) = pack4(a0, b0, c0, d0);
  int sx = X0 + X1 + X2 + X3;                  // |sum over the block| < 2^31
  sx += __shfl_xor_sync(0xffffffffu, sx, 1);
  sx += __shfl_xor_sync(0xffffffffu, sx, 2);
  sx += __shfl_xor_sync(0xffffffffu, sx, 4);
  if ((lane & 7) == 0) lsc_vec[blk] = make_float2(s, __fmul_rn(s, (float)sx));
}

struct Acc {
  float r0[4], r1[4];  // rows g / g+8 x column groups q
};

// Dot products of one 16-row tile (K = 32 * nblk, nblk % 4 == 0) with n <= NP
// activation vectors (vector ids vid[0..n)). Returns the lane's share; see the
// file header for the column layout. Not inlined: phase 1 and phase 2 share one
// copy of the code, which keeps the instruction footprint small.
//   NP = 1: one accumulator tile holds 2 blocks of the token (2 tiles per chunk)
//   NP >= 2: one tile holds 2 tokens of one block; NQ = NP/2 tiles per block
// Every variant forms a token's result in the same floating-point order: the
// blocks of even and of odd index accumulate separately (in increasing block
// order, each half of a limb pair on its own lane), the two halves are added,
// then even + odd. So a token's output does not depend on how many tokens of
// the batch share the expert (NP), and a verify batch reproduces single-token
// decoding bit for bit.
template <int BITS, int NP>
__device__ __noinline__ Acc tile_dot(const uint8_t *tile, int nblk, const uint8_t *limbs, const float2 *lsc,
                                     const int *vid, int n) {
  constexpr int TS = NP == 1 ? 1 : 2;     // tokens per accumulator tile
  constexpr int BS = 2 / TS;              // blocks per accumulator tile
  constexpr int NQ = NP == 1 ? 1 : NP / 2;
  constexpr int NSET = 4 / BS;            // tiles per 4-block chunk and column group
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  // B columns this lane provides: column g -> pair g>>2, limb slot g&3 (l2, l1, zero, l0)
  const int pP = g >> 2, pslot = g & 3;
  const int ploff = pslot == 0 ? 0 : (pslot == 1 ? 32 : 64);
  // D columns this lane reads: (2t, 2t+1) -> pair t>>1, half t&1
  const int oP = t >> 1, ohalf = t & 1;
  const float wgt = ohalf ? 1.0f : 256.0f;
  const uint8_t *sbase = tile + 64 * nblk * BITS;   // scales follow the codes
  float acc[2][NQ];
  float acc_odd[2][NQ];   // NP >= 2: odd blocks (for NP == 1 the lanes of pair 1 hold them)
  int pv[NQ], ov[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    acc[0][q] = acc[1][q] = 0.0f;
    acc_odd[0][q] = acc_odd[1][q] = 0.0f;
    const int ptq = (NP == 1) ? 0 : 2 * q + pP;
    const int otq = (NP == 1) ? 0 : 2 * q + oP;
    pv[q] = (ptq < n && pslot != 2) ? vid[ptq] : -1;
    ov[q] = otq < n ? vid[otq] : -1;
  }
  const int pbeta = (NP == 1) ? pP : 0;
  const int obeta = (NP == 1) ? oP : 0;

#pragma unroll 1
  for (int c = 0; c < (nblk >> 2); ++c) {
    uint32_t w[8];
    if (BITS == 2) {
      const uint4 q = *reinterpret_cast<const uint4 *>(tile + c * 512 + lane * 16);
      w[0] = q.x; w[1] = q.y; w[2] = q.z; w[3] = q.w;
    } else {
      const uint4 q0 = *reinterpret_cast<const uint4 *>(tile + (2 * c) * 512 + lane * 16);
      const uint4 q1 = *reinterpret_cast<const uint4 *>(tile + (2 * c + 1) * 512 + lane * 16);
      w[0] = q0.x; w[1] = q0.y; w[2] = q0.z; w[3] = q0.w;
      w[4] = q1.x; w[5] = q1.y; w[6] = q1.z; w[7] = q1.w;
    }
    // all MMAs of the chunk first, into separate accumulators, then their
    // epilogues in the same (sb, q) order as before: the MMA latency overlaps
    // (a warp keeps NSET x NQ x BS of them in flight instead of one) and the
    // floating-point order of the results is unchanged
    uint32_t bq[NSET][NQ][2];
#pragma unroll
    for (int sb = 0; sb < NSET; ++sb)
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        // lanes without a token (or on the zero limb column) read vector 0's
        // record, in bounds, and pass zeros
        const int blk = c * 4 + sb * BS + pbeta;
        const int pvs = pv[q] >= 0 ? pv[q] : vid[0];
        const uint8_t *lp = limbs + ((size_t)pvs * nblk + blk) * LIMB_REC + ploff + 4 * t;
        const uint32_t x0 = *reinterpret_cast<const uint32_t *>(lp);
        const uint32_t x1 = *reinterpret_cast<const uint32_t *>(lp + 16);
        bq[sb][q][0] = pv[q] >= 0 ? x0 : 0u;
        bq[sb][q][1] = pv[q] >= 0 ? x1 : 0u;
      }
    int D[NSET][NQ][4];
#pragma unroll
    for (int sb = 0; sb < NSET; ++sb)
#pragma unroll
      for (int q = 0; q < NQ; ++q) D[sb][q][0] = D[sb][q][1] = D[sb][q][2] = D[sb][q][3] = 0;
#pragma unroll
    for (int beta = 0; beta < BS; ++beta)
#pragma unroll
      for (int sb = 0; sb < NSET; ++sb) {
        const int bb = sb * BS + beta;
        uint32_t a0, a1, a2, a3;
        if (BITS == 2) {
          const uint32_t x = w[bb];
          a0 = x & 0x03030303u;
          a1 = (x >> 2) & 0x03030303u;
          a2 = (x >> 4) & 0x03030303u;
          a3 = (x >> 6) & 0x03030303u;
        } else {
          const uint32_t x0 = w[2 * bb], x1 = w[2 * bb + 1];
          a0 = x0 & 0x0F0F0F0Fu;
          a1 = (x0 >> 4) & 0x0F0F0F0Fu;
          a2 = x1 & 0x0F0F0F0Fu;
          a3 = (x1 >> 4) & 0x0F0F0F0Fu;
        }
        const bool on = (pbeta == beta);
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          mma_u8s8(D[sb][q][0], D[sb][q][1], D[sb][q][2], D[sb][q][3], a0, a1, a2, a3, on ? bq[sb][q][0] : 0u,
                   on ? bq[sb][q][1] : 0u);
      }
#pragma unroll
    for (int sb = 0; sb < NSET; ++sb)
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        if (ov[q] >= 0) {
          const int bo = c * 4 + sb * BS + obeta;
          const float v0 = limb_pair_b<BITS>(D[sb][q][0], D[sb][q][1]);
          const float v1 = limb_pair_b<BITS>(D[sb][q][2], D[sb][q][3]);
          const float2 ss = lsc[(size_t)ov[q] * nblk + bo];
          const uint2 dm = *reinterpret_cast<const uint2 *>(sbase + (bo * 8 + g) * 8);
          const float sw = ss.x * wgt;
          const float mt = ohalf ? 0.0f : ss.y;    // the min term once per pair
          if (NP == 1 || (bo & 1) == 0) {
            acc[0][q] = fmaf(h2f(dm.x & 0xffffu), sw * v0, fmaf(h2f(dm.x >> 16), mt, acc[0][q]));
            acc[1][q] = fmaf(h2f(dm.y & 0xffffu), sw * v1, fmaf(h2f(dm.y >> 16), mt, acc[1][q]));
          } else {
            acc_odd[0][q] = fmaf(h2f(dm.x & 0xffffu), sw * v0, fmaf(h2f(dm.x >> 16), mt, acc_odd[0][q]));
            acc_odd[1][q] = fmaf(h2f(dm.y & 0xffffu), sw * v1, fmaf(h2f(dm.y >> 16), mt, acc_odd[1][q]));
          }
        }
      }
  }
  // combine the lanes that share a token: the two halves of a pair, then even
  // + odd blocks (for NP == 1 the other pair of lanes, else acc_odd)
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      acc[r][q] += __shfl_xor_sync(0xffffffffu, acc[r][q], 1);
      if (NP == 1) {
        acc[r][q] += __shfl_xor_sync(0xffffffffu, acc[r][q], 2);
      } else {
        acc_odd[r][q] += __shfl_xor_sync(0xffffffffu, acc_odd[r][q], 1);
        acc[r][q] += acc_odd[r][q];
      }
    }
  }
  Acc out;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    out.r0[q] = q < NQ ? acc[0][q < NQ ? q : 0] : 0.0f;
    out.r1[q] = q < NQ ? acc[1][q < NQ ? q : 0] : 0.0f;
  }
  return out;
}

template <int BITS>
__device__ __forceinline__ int dispatch_dot(const uint8_t *tile, int nblk, const uint8_t *limbs, const float2 *lsc,
                                            const int *vid, int n, Acc &acc) {
  if (n <= 1) { acc = tile_dot<BITS, 1>(tile, nblk, limbs, lsc, vid, n); return 1; }
  if (n <= 2) { acc = tile_dot<BITS, 2>(tile, nblk, limbs, lsc, vid, n); return 2; }
  if (n <= 4) { acc = tile_dot<BITS, 4>(tile, nblk, limbs, lsc, vid, n); return 4; }
  acc = tile_dot<BITS, 8>(tile, nblk, limbs, lsc, vid, n);
  return 8;
}

// Token held by lane t in column group q after tile_dot (or -1): lane 0 for
// NP == 1; for NP >= 2 lanes 0 and 2 hold tokens 2q and 2q + 1.
__device__ __forceinline__ int owner(int np, int t, int q) {
  if (np == 1) return (t == 0 && q == 0) ? 0 : -1;
  if (t & 1) return -1;
  return q < np / 2 ? 2 * q + (t >> 1) : -1;
}

// Single-vector variant of tile_dot (NP == 1) with NCH 4-block chunks in flight,
// so that independent MMAs and shared-memory loads overlap. Returns the tile's
// rows (g, g+8) dot products; every lane of a quad holds them after the final
// reduction. `limbs` / `lsc` point at the activation vector's own records.
template <int BITS, int NCH = 2>
__device__ __noinline__ float2 tile_dot1(const uint8_t *tile, int nblk, const uint8_t *limbs, const float2 *lsc) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int pP = g >> 2, pslot = g & 3;
  const int ploff = pslot == 0 ? 0 : (pslot == 1 ? 32 : 64);
  const bool pon = pslot != 2;
  const int oP = t >> 1, ohalf = t & 1;
  const float wgt = ohalf ? 1.0f : 256.0f;
  const uint8_t *sbase = tile + 64 * nblk * BITS;
  const int nchunks = nblk >> 2;
  float acc0 = 0.0f, acc1 = 0.0f;
  for (int c0 = 0; c0 < nchunks; c0 += NCH) {
    uint32_t w[NCH][8];
    uint32_t bv[NCH][2][2];
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      const int c = c0 + ch;
      if (c < nchunks) {
        if (BITS == 2) {
          const uint4 q = *reinterpret_cast<const uint4 *>(tile + c * 512 + lane * 16);
          w[ch][0] = q.x; w[ch][1] = q.y; w[ch][2] = q.z; w[ch][3] = q.w;
        } else {
          const uint4 q0 = *reinterpret_cast<const uint4 *>(tile + (2 * c) * 512 + lane * 16);
          const uint4 q1 = *reinterpret_cast<const uint4 *>(tile + (2 * c + 1) * 512 + lane * 16);
          w[ch][0] = q0.x; w[ch][1] = q0.y; w[ch][2] = q0.z; w[ch][3] = q0.w;
          w[ch][4] = q1.x; w[ch][5] = q1.y; w[ch][6] = q1.z; w[ch][7] = q1.w;
        }
#pragma unroll
        for (int sb = 0; sb < 2; ++sb) {
          bv[ch][sb][0] = bv[ch][sb][1] = 0u;
          if (pon) {
            const uint8_t *lp = limbs + (size_t)(c * 4 + sb * 2 + pP) * LIMB_REC + ploff + 4 * t;
            bv[ch][sb][0] = *reinterpret_cast<const uint32_t *>(lp);
            bv[ch][sb][1] = *reinterpret_cast<const uint32_t *>(lp + 16);
          }
        }
      }
    }
    int D[NCH][2][4];
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
      for (int sb = 0; sb < 2; ++sb) D[ch][sb][0] = D[ch][sb][1] = D[ch][sb][2] = D[ch][sb][3] = 0;
#pragma unroll
    for (int beta = 0; beta < 2; ++beta) {
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        if (c0 + ch < nchunks) {
#pragma unroll
          for (int sb = 0; sb < 2; ++sb) {
            const int bb = sb * 2 + beta;
            uint32_t a0, a1, a2, a3;
            if (BITS == 2) {
              const uint32_t x = w[ch][bb];
              a0 = x & 0x03030303u;
              a1 = (x >> 2) & 0x03030303u;
              a2 = (x >> 4) & 0x03030303u;
              a3 = (x >> 6) & 0x03030303u;
            } else {
              const uint32_t x0 = w[ch][2 * bb], x1 = w[ch][2 * bb + 1];
              a0 = x0 & 0x0F0F0F0Fu;
              a1 = (x0 >> 4) & 0x0F0F0F0Fu;
              a2 = x1 & 0x0F0F0F0Fu;
              a3 = (x1 >> 4) & 0x0F0F0F0Fu;
            }
            const bool on = pP == beta;
            mma_u8s8(D[ch][sb][0], D[ch][sb][1], D[ch][sb][2], D[ch][sb][3], a0, a1, a2, a3,
                     on ? bv[ch][sb][0] : 0u, on ? bv[ch][sb][1] : 0u);
          }
        }
      }
    }
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      if (c0 + ch < nchunks) {
#pragma unroll
        for (int sb = 0; sb < 2; ++sb) {
          const int bo = (c0 + ch) * 4 + sb * 2 + oP;
          const float v0 = limb_pair_b<BITS>(D[ch][sb][0], D[ch][sb][1]);
          const float v1 = limb_pair_b<BITS>(D[ch][sb][2], D[ch][sb][3]);
          const float2 ss = lsc[bo];
          const uint2 dm = *reinterpret_cast<const uint2 *>(sbase + (bo * 8 + g) * 8);
          const float sw = ss.x * wgt;
          const float mt = ohalf ? 0.0f : ss.y;
          acc0 = fmaf(h2f(dm.x & 0xffffu), sw * v0, fmaf(h2f(dm.x >> 16), mt, acc0));
          acc1 = fmaf(h2f(dm.y & 0xffffu), sw * v1, fmaf(h2f(dm.y >> 16), mt, acc1));
        }
      }
    }
  }
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 1);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 1);
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 2);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 2);
  return make_float2(acc0, acc1);
}

// Inline form of quant_chunk, for loops whose iterations the compiler may
// interleave. s and inv need not be exact inverses: the contraction uses s
// itself, so s * X still tracks v to within rounding of the quantisation.
__device__ __forceinline__ void quant_chunk_inl(float4 v, uint8_t *limbs_vec, float2 *lsc_vec, int chunk, int lane) {
  float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
  float s, inv;
  block_scale(a, s, inv);
  const int X0 = quant_one(v.x, inv), X1 = quant_one(v.y, inv), X2 = quant_one(v.z, inv), X3 = quant_one(v.w, inv);
  int a2, a1, a0, b2, b1, b0, c2, c1, c0, d2, d1, d0;
  limbs3(X0, a2, a1, a0);
  limbs3(X1, b2, b1, b0);
  limbs3(X2, c2, c1, c0);
  limbs3(X3, d2, d1, d0);
  const int blk = chunk * 4 + (lane >> 3);
  uint8_t *rec = limbs_vec + (size_t)blk * LIMB_REC + (lane & 7) * 4;
  *reinterpret_cast<uint32_t *>(rec) = pack4(a2, b2, c2, d2);
  *reinterpret_cast<uint32_t *>(rec + 32) = pack4(a1, b1, c1, d1);
  *reinterpret_cast<uint32_t *>(rec + 64) = pack4(a0, b0, c0, d0);
  int sx = X0 + X1 + X2 + X3;
  sx += __shfl_xor_sync(0xffffffffu, sx, 1);
  sx += __shfl_xor_sync(0xffffffffu, sx, 2);
  sx += __shfl_xor_sync(0xffffffffu, sx, 4);
  if ((lane & 7) == 0) lsc_vec[blk] = make_float2(s, __fmul_rn(s, (float)sx));
}

// Two chunks (see quant_chunk) in one call.
__device__ __noinline__ void quant_chunk2(float4 v0, uint8_t *limbs0, float2 *lsc0, int chunk0, float4 v1,
                                          uint8_t *limbs1, float2 *lsc1, int chunk1, int lane) {
  quant_chunk_inl(v0, limbs0, lsc0, chunk0, lane);
  quant_chunk_inl(v1, limbs1, lsc1, chunk1, lane);
}

// Quantise activation vectors of 128-element chunks; task = vec * nch + chunk.
// Each warp first issues the loads of up to MB tasks, then quantises them, so a
// warp pays one memory latency per MB tasks.
template <int NW, int MB, typename Load>
__device__ __forceinline__ void quant_tasks(int ntask, int nch, int nblk, uint8_t *limbs, float2 *lsc, int warp,
                                            int lane, Load load) {
  for (int base = warp; base < ntask; base += MB * NW) {
    float4 v[MB];
#pragma unroll
    for (int i = 0; i < MB; ++i) {
      const int task = base + i * NW;
      if (task < ntask) v[i] = load(task / nch, task % nch);
    }
    // two chunks a call, so that their shuffle chains overlap
#pragma unroll
    for (int i = 0; i < MB; i += 2) {
      const int t0 = base + i * NW, t1 = base + (i + 1) * NW;
      if (t0 < ntask) {
        const int u1 = t1 < ntask ? t1 : t0;   // a lone chunk is quantised twice into the same place
        quant_chunk2(v[i], limbs + (size_t)(t0 / nch) * nblk * LIMB_REC, lsc + (size_t)(t0 / nch) * nblk, t0 % nch,
                     t1 < ntask ? v[i + 1] : v[i], limbs + (size_t)(u1 / nch) * nblk * LIMB_REC,
                     lsc + (size_t)(u1 / nch) * nblk, u1 % nch, lane);
      }
    }
  }
}



}  // namespace
}  // namespace tile
}  // namespace qmoe
