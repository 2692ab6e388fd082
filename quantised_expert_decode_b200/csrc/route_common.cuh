// Warp-level top-k selection with renormalised gates over one token's float64
// logits (used by the decode and prefill routers).
//
// Selection order: logit descending, expert index ascending on equal logits.
// 1. Every logit gets an fp32 key (round-to-nearest of the float64 value, -0
//    taken as +0, made order-preserving as an unsigned integer). Rounding is
//    monotone and equal logits get equal keys, so the k largest float64
//    logits are among the k largest keys, counted with multiplicity.
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
    const float f = __double2float_rn(val[j]);
    key[j] = e < E ? float_key(f == 0.0f ? 0.0f : f) : 0u;
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
  if (total <= TOPK_CAND) {
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
