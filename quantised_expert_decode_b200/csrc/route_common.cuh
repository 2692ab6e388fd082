// Warp-level top-k selection with renormalised gates over one token's float64
// logits (used by the decode and prefill routers).
//
// Selection order: logit descending, expert index ascending on equal logits.
// 1. Every logit gets a 32-bit key: the top half of the float64 value's bits
//    made order-preserving as an unsigned integer (-0 taken as +0). Dropping
//    the low bits is monotone and equal logits get equal keys, so the k
//    largest float64 logits are among the k largest keys, counted with
//    multiplicity. (Integer operations only: a float64 -> float32 rounding
//    would issue on the conversion unit, which runs at a fraction of the rate.)
// 2. Threshold: the k-th largest of the 32 per-lane maximum keys (ties by
//    lane). At least k keys (those lane maxima) are >= it, so it is at most
//    the k-th largest key and every key >= threshold is a candidate: a
//    superset of the k largest. One pass of 32 independent shuffles ranks the
//    lane maxima, instead of k dependent rounds of warp reductions.
// 3. Candidates are ranked exactly on their float64 logits (index breaks
//    ties). Ranks below k give the slots.
// 4. gate_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0) over the selected slots.
#pragma once

#include "common.cuh"

namespace qmoe {

constexpr int TOPK_MAX_K = 16;
constexpr int TOPK_CAND = 64;

struct TopkScratch {
  int cand[TOPK_CAND];
  double cand_v[TOPK_CAND];
  int sel_e[TOPK_MAX_K];
  double sel_v[TOPK_MAX_K];
};

__device__ __forceinline__ unsigned double_key(double v) {
  const long long b = __double_as_longlong(v == 0.0 ? 0.0 : v);
  const unsigned long long o = b < 0 ? ~(unsigned long long)b : ((unsigned long long)b | 0x8000000000000000ull);
  return (unsigned)(o >> 32);
}

__device__ __forceinline__ bool ranks_above(double va, int ea, double vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

// A NaN logit ranks as -infinity, so the ranking is a total order and the k
// selected slots are always k distinct valid experts.
__device__ __forceinline__ double rank_value(double v) { return isnan(v) ? -INFINITY : v; }

// One warp; get(e) returns the token's float64 logit of expert e (global
// memory written by other CTAs and read through L2, or shared memory).
// M = values per lane = ceil(E / 32).
template <int M, typename Get>
__device__ inline void warp_topk_gates_m(Get get, int E, int k, int32_t *idx_out, float *gate_out,
                                         TopkScratch *sc) {
  const int lane = threadIdx.x & 31;
  double val[M];
  unsigned key[M];
#pragma unroll
  for (int j = 0; j < M; ++j) {
    const int e = lane + 32 * j;
    val[j] = e < E ? rank_value(get(e)) : 0.0;
  }
#pragma unroll
  for (int j = 0; j < M; ++j) {
    const int e = lane + 32 * j;
    // -0 and +0 are equal logits (ranked by index), so they share one key
    key[j] = e < E ? double_key(val[j]) : 0u;
  }
  unsigned lmax = 0;
#pragma unroll
  for (int j = 0; j < M; ++j) lmax = max(lmax, key[j]);
  int rank = 0;   // lanes whose maximum ranks above this lane's
#pragma unroll
  for (int s2 = 0; s2 < 32; ++s2) {
    const unsigned o = __shfl_sync(0xffffffffu, lmax, s2);
    rank += (o > lmax || (o == lmax && s2 < lane)) ? 1 : 0;
  }
  // ranks are a permutation of 0..31; k <= TOPK_MAX_K <= 32. Lanes without a
  // valid key have maximum 0, so with fewer than k such lanes thr is 0 and
  // every valid key is a candidate.
  const unsigned at = __ballot_sync(0xffffffffu, rank == k - 1);
  const unsigned thr = __shfl_sync(0xffffffffu, lmax, __ffs(at) - 1);
  // candidates: keys >= thr
  int mine = 0;
#pragma unroll
  for (int j = 0; j < M; ++j) mine += (key[j] != 0u && key[j] >= thr) ? 1 : 0;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total <= 32) {
    // one candidate per lane (in lane order of the keys), ranked against the
    // others through shuffles
    int pos = incl - mine, ce = 0;
    double cv = 0.0;
#pragma unroll
    for (int j = 0; j < M; ++j)
      if (key[j] != 0u && key[j] >= thr) {
        sc->cand[pos] = lane + 32 * j;
        sc->cand_v[pos] = val[j];
        ++pos;
      }
    __syncwarp();
    if (lane < total) {
      ce = sc->cand[lane];
      cv = sc->cand_v[lane];
    }
    int rank = 0;
#pragma unroll
    for (int i2 = 0; i2 < 32; ++i2) {   // all 32 shuffles independent; lanes past `total` hold no candidate
      const double v2 = __shfl_sync(0xffffffffu, cv, i2);
      const int e2 = __shfl_sync(0xffffffffu, ce, i2);
      rank += (i2 < total && ranks_above(v2, e2, cv, ce)) ? 1 : 0;
    }
    if (lane < total && rank < k) {
      sc->sel_e[rank] = ce;
      sc->sel_v[rank] = cv;
    }
  } else if (total <= TOPK_CAND) {
    int pos = incl - mine;
#pragma unroll
    for (int j = 0; j < M; ++j)
      if (key[j] != 0u && key[j] >= thr) {
        sc->cand[pos] = lane + 32 * j;
        sc->cand_v[pos] = val[j];
        ++pos;
      }
    __syncwarp();
    for (int i = lane; i < total; i += 32) {
      const int e = sc->cand[i];
      const double v = sc->cand_v[i];
      int rank = 0;
      for (int i2 = 0; i2 < total; ++i2) rank += ranks_above(sc->cand_v[i2], sc->cand[i2], v, e) ? 1 : 0;
      if (rank < k) {
        sc->sel_e[rank] = e;
        sc->sel_v[rank] = v;
      }
    }
  } else {
    // many equal fp32 keys (degenerate router): rank the candidates against all logits
#pragma unroll
    for (int j = 0; j < M; ++j) {
      if (key[j] != 0u && key[j] >= thr) {
        const int e = lane + 32 * j;
        const double v = val[j];
        int rank = 0;
        for (int e2 = 0; e2 < E && rank < k; ++e2) rank += ranks_above(rank_value(get(e2)), e2, v, e) ? 1 : 0;
        if (rank < k) {
          sc->sel_e[rank] = e;
          sc->sel_v[rank] = v;
        }
      }
    }
  }
  __syncwarp();
  float ex = 0.0f;
  if (lane < k) ex = expf((float)(sc->sel_v[lane] - sc->sel_v[0]));
  const float sum = warp_sum(ex);
  if (lane < k) {
    idx_out[lane] = sc->sel_e[lane];
    gate_out[lane] = ex / sum;
  }
  __syncwarp();
}

// Key of a float64 logit from its bits: the high word made order-preserving
// as an unsigned integer. Every negative number whose high word is
// 0x80000000 (-0 and the smallest subnormals) takes the key of +0, which keeps
// the key monotone and gives -0 and +0 one key; NaN takes the key of
// -infinity, its rank. Integer operations only; never 0 (0 marks "no logit").
__device__ __forceinline__ unsigned logit_key(double v) {
  unsigned hi = (unsigned)__double2hiint(v);
  const unsigned ahi = hi & 0x7fffffffu;
  if (ahi >= 0x7ff00000u && (ahi > 0x7ff00000u || (unsigned)__double2loint(v) != 0u)) hi = 0xfff00000u;
  if (hi == 0x80000000u) hi = 0u;
  return hi ^ ((unsigned)((int)hi >> 31) | 0x80000000u);
}

// Position of expert e's key in a per-lane key table of M keys a lane
// (lane e % 32 holds the keys of experts e % 32 + 32 j, j < M, contiguously).
__device__ __forceinline__ int key_slot(int e, int M) { return (e & 31) * M + (e >> 5); }

// Keys per lane for E experts (a power of two, at least 4 so that a lane's
// keys load as 16-byte vectors).
__host__ __device__ constexpr int topk_m(int E) {
  return E <= 128 ? 4 : E <= 256 ? 8 : E <= 512 ? 16 : 32;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// The selection above with the keys already in registers: lane l holds
// key[j] = key of expert l + 32 j (0 for e >= E), and val(e) returns expert
// e's float64 logit (for the candidates only). Candidate positions come from
// one ballot per key column, so no step waits on a chain of shuffles.
// COMPACT keeps the shuffle loops rolled: for a selection that runs once per
// launch, the instruction fetches of unrolled code cost more than the loop.
template <int M, bool COMPACT = false, class Val>
__device__ __forceinline__ void warp_topk_keys(const unsigned (&key)[M], Val val, int E, int k, int32_t *idx_out,
                                               float *gate_out, TopkScratch *sc) {
  const int lane = threadIdx.x & 31;
  unsigned lmax = key[0];
#pragma unroll
  for (int j = 1; j < M; ++j) lmax = max(lmax, key[j]);
  int rank = 0;
#pragma unroll(COMPACT ? 1 : 32)
  for (int s2 = 0; s2 < 32; ++s2) {
    const unsigned o = __shfl_sync(0xffffffffu, lmax, s2);
    rank += (o > lmax || (o == lmax && s2 < lane)) ? 1 : 0;
  }
  // ranks are a permutation of 0..31; k <= TOPK_MAX_K <= 32. Lanes without a
  // valid key have maximum 0, so with fewer than k such lanes thr is 0 and
  // every valid key is a candidate.
  const unsigned at = __ballot_sync(0xffffffffu, rank == k - 1);
  const unsigned thr = __shfl_sync(0xffffffffu, lmax, __ffs(at) - 1);
  const unsigned below = lanemask_lt();
  int total = 0;
#pragma unroll
  for (int j = 0; j < M; ++j) {
    const bool c = key[j] != 0u && key[j] >= thr;
    const unsigned b = __ballot_sync(0xffffffffu, c);
    const int pos = total + __popc(b & below);
    if (c && pos < TOPK_CAND) sc->cand[pos] = lane + 32 * j;
    total += __popc(b);
  }
  __syncwarp();
  if (total <= 32) {
    int ce = 0;
    double cv = 0.0;
    if (lane < total) {
      ce = sc->cand[lane];
      cv = rank_value(val(ce));
    }
    int r = 0;
    if (total <= 16) {
#pragma unroll(COMPACT ? 1 : 16)
      for (int i2 = 0; i2 < 16; ++i2) {
        const double v2 = __shfl_sync(0xffffffffu, cv, i2);
        const int e2 = __shfl_sync(0xffffffffu, ce, i2);
        r += (i2 < total && ranks_above(v2, e2, cv, ce)) ? 1 : 0;
      }
    } else {
#pragma unroll(COMPACT ? 1 : 32)
      for (int i2 = 0; i2 < 32; ++i2) {
        const double v2 = __shfl_sync(0xffffffffu, cv, i2);
        const int e2 = __shfl_sync(0xffffffffu, ce, i2);
        r += (i2 < total && ranks_above(v2, e2, cv, ce)) ? 1 : 0;
      }
    }
    if (lane < total && r < k) {
      sc->sel_e[r] = ce;
      sc->sel_v[r] = cv;
    }
  } else if (total <= TOPK_CAND) {
    for (int i = lane; i < total; i += 32) sc->cand_v[i] = rank_value(val(sc->cand[i]));
    __syncwarp();
    for (int i = lane; i < total; i += 32) {
      const int e = sc->cand[i];
      const double v = sc->cand_v[i];
      int r = 0;
      for (int i2 = 0; i2 < total; ++i2) r += ranks_above(sc->cand_v[i2], sc->cand[i2], v, e) ? 1 : 0;
      if (r < k) {
        sc->sel_e[r] = e;
        sc->sel_v[r] = v;
      }
    }
  } else {
    // many equal keys (degenerate router): rank the candidates against all logits
#pragma unroll
    for (int j = 0; j < M; ++j) {
      if (key[j] != 0u && key[j] >= thr) {
        const int e = lane + 32 * j;
        const double v = rank_value(val(e));
        int r = 0;
        for (int e2 = 0; e2 < E && r < k; ++e2) r += ranks_above(rank_value(val(e2)), e2, v, e) ? 1 : 0;
        if (r < k) {
          sc->sel_e[r] = e;
          sc->sel_v[r] = v;
        }
      }
    }
  }
  __syncwarp();
  float ex = 0.0f;
  if (lane < k) ex = expf((float)(sc->sel_v[lane] - sc->sel_v[0]));
  const float sum = warp_sum(ex);
  if (lane < k) {
    idx_out[lane] = sc->sel_e[lane];
    gate_out[lane] = ex / sum;
  }
  __syncwarp();
}

// Selection from float64 logits lg[0, E) and their keys in a per-lane key
// table (key_slot layout, M = topk_m(E) keys a lane), both in shared memory.
template <int M>
__device__ __forceinline__ void warp_topk_table_m(const double *lg, const unsigned *keys, int E, int k,
                                                  int32_t *idx_out, float *gate_out, TopkScratch *sc) {
  const int lane = threadIdx.x & 31;
  unsigned key[M];
#pragma unroll
  for (int q = 0; q < M / 4; ++q) {
    const uint4 v = reinterpret_cast<const uint4 *>(keys + lane * M)[q];
    key[4 * q] = v.x; key[4 * q + 1] = v.y; key[4 * q + 2] = v.z; key[4 * q + 3] = v.w;
  }
#pragma unroll
  for (int j = 0; j < M; ++j)
    if (lane + 32 * j >= E) key[j] = 0u;
  warp_topk_keys<M>(key, [&](int e) { return lg[e]; }, E, k, idx_out, gate_out, sc);
}

template <typename Get>
__device__ inline void warp_topk_gates_get(Get get, int E, int k, int32_t *idx_out, float *gate_out,
                                           TopkScratch *sc) {
  if (E <= 32) warp_topk_gates_m<1>(get, E, k, idx_out, gate_out, sc);
  else if (E <= 64) warp_topk_gates_m<2>(get, E, k, idx_out, gate_out, sc);
  else if (E <= 128) warp_topk_gates_m<4>(get, E, k, idx_out, gate_out, sc);
  else if (E <= 256) warp_topk_gates_m<8>(get, E, k, idx_out, gate_out, sc);
  else if (E <= 512) warp_topk_gates_m<16>(get, E, k, idx_out, gate_out, sc);
  else warp_topk_gates_m<32>(get, E, k, idx_out, gate_out, sc);
}

// Logits in global memory, written by other CTAs of this grid before a fence.
__device__ inline void warp_topk_gates(const double *l, int E, int k, int32_t *idx_out, float *gate_out,
                                       TopkScratch *sc) {
  warp_topk_gates_get([&](int e) { return __ldcg(l + e); }, E, k, idx_out, gate_out, sc);
}

}  // namespace qmoe
