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
