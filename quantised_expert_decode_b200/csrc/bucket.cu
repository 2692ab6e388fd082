// Token -> expert bucketing for prefill chunks: a stable counting sort of the
// (token, slot) pairs by expert. Pairs are numbered p = t*k + j; the sorted
// order is (expert, t, j), so the permutation is unique and reproducible.
//
// Two launches over C CTAs, CTA c owning a contiguous run of whole tokens:
//   bk_count: per-CTA expert histogram -> table cnt[c][e] (and a per-CTA
//             error flag: index out of range, or an expert repeated within
//             one token's route when that check is on);
//   bk_place: every CTA reads the table for all experts, so it knows both the
//             global offsets (exclusive prefix of the column sums over e) and
//             its own base per expert (plus the counts of CTAs before it);
//             it then recounts its pairs per warp and places them in pair
//             order. No CTA waits on another.
#include <algorithm>

#include "common.cuh"

namespace qmoe {
namespace {

constexpr int BK_MAX_E = 1024;
constexpr int BK_MAX_CTAS = 148;       // one CTA per SM at most
constexpr int BK_MIN_TOKENS = 64;      // tokens per CTA below which more CTAs only add table reads
constexpr int BK_COUNT_THREADS = 256;
constexpr int BK_PLACE_THREADS = 512;  // thread i owns experts 2i and 2i+1 in the scans
constexpr int BK_PLACE_WARPS = BK_PLACE_THREADS / 32;

struct BucketArgs {
  const int32_t *idx;   // [P]
  const float *gate;    // [P] or null
  int T, k, E, C;
  int32_t *cnt;         // [C][E] workspace: per-CTA expert counts
  int32_t *flag;        // [C] workspace: per-CTA error code (0 = none)
  int32_t *offsets;     // [E + 1]
  int32_t *perm;        // [P] sorted position -> pair id
  int32_t *ptok;        // [P] or null: token of each sorted pair
  float *pgate;         // [P] or null: gate of each sorted pair
  int32_t *active;      // [E] or null: experts with at least one pair, ascending
  int32_t *nactive;     // [1] or null
  int check_dup;        // report an expert repeated within one token's route
  int32_t *status;
};

// pairs [lo, hi) of CTA c: the pairs of tokens [c*T/C, (c+1)*T/C)
__device__ __forceinline__ void cta_pairs(const BucketArgs &a, int c, int &lo, int &hi) {
  lo = (int)((long long)c * a.T / a.C) * a.k;
  hi = (int)((long long)(c + 1) * a.T / a.C) * a.k;
}

__global__ void __launch_bounds__(BK_COUNT_THREADS) bk_count_kernel(BucketArgs a) {
  extern __shared__ int hist[];   // [E]
  __shared__ int bad;
  const int tid = threadIdx.x, c = blockIdx.x, E = a.E;
  for (int i = tid; i < E; i += BK_COUNT_THREADS) hist[i] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  int lo, hi;
  cta_pairs(a, c, lo, hi);
  // four pairs per thread per step, loads issued before use
  for (int p0 = lo + tid; p0 < hi; p0 += 4 * BK_COUNT_THREADS) {
    int ev[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + u * BK_COUNT_THREADS;
      ev[u] = p < hi ? a.idx[p] : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + u * BK_COUNT_THREADS;
      if (p >= hi) continue;
      const int e = ev[u];
      if (e < 0 || e >= E) {
        bad = DEV_BAD_INDEX;
        continue;
      }
      if (a.check_dup) {
        const int j = p % a.k;
        for (int j2 = 0; j2 < j; ++j2)
          if (a.idx[p - j + j2] == e) bad = DEV_DUP_INDEX;
      }
      atomicAdd(&hist[e], 1);
    }
  }
  __syncthreads();
  for (int i = tid; i < E; i += BK_COUNT_THREADS) a.cnt[(size_t)c * E + i] = hist[i];
  if (tid == 0) {
    a.flag[c] = bad;
    if (bad) set_status(a.status, bad);
  }
}

__global__ void __launch_bounds__(BK_PLACE_THREADS, 1) bk_place_kernel(BucketArgs a) {
  extern __shared__ int hist[];   // [BK_PLACE_WARPS][E]: counts, then running positions
  __shared__ int wtot[2][BK_PLACE_WARPS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, c = blockIdx.x;
  const int E = a.E, C = a.C;
  int f = 0;
  for (int i = tid; i < C; i += BK_PLACE_THREADS) f |= a.flag[i];
  if (__syncthreads_or(f)) return;   // the count kernel has set the status; outputs stay unwritten
  for (int i = tid; i < BK_PLACE_WARPS * E; i += BK_PLACE_THREADS) hist[i] = 0;

  // column sums of the table for experts 2*tid, 2*tid+1: before this CTA, and over all CTAs
  int before[2] = {0, 0}, tot[2] = {0, 0};
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    if (e >= E) continue;
    const int32_t *col = a.cnt + e;
    for (int c0 = 0; c0 < C; c0 += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = c0 + u < C ? col[(size_t)(c0 + u) * E] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        tot[r] += v[u];
        if (c0 + u < c) before[r] += v[u];
      }
    }
  }
  // block-wide exclusive scans of pair counts and active flags over experts
  const int v = tot[0] + tot[1];
  const int fl = (tot[0] > 0) + (tot[1] > 0);
  int iv = v, ifl = fl, dummy = 0;
  warp_scan3(iv, ifl, dummy);
  if (lane == 31) {
    wtot[0][warp] = iv;
    wtot[1][warp] = ifl;
  }
  __syncthreads();   // also orders the hist zeroing before pass 1
  if (warp == 0) {
    const int s0 = lane < BK_PLACE_WARPS ? wtot[0][lane] : 0, s1 = lane < BK_PLACE_WARPS ? wtot[1][lane] : 0;
    int i0 = s0, i1 = s1, s2 = 0;
    warp_scan3(i0, i1, s2);
    if (lane < BK_PLACE_WARPS) {
      wtot[0][lane] = i0 - s0;
      wtot[1][lane] = i1 - s1;
    }
  }
  __syncthreads();
  int off = wtot[0][warp] + iv - v;
  int act = wtot[1][warp] + ifl - fl;
  int base[2];
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    base[r] = off + before[r];
    if (e < E && c == 0) {
      a.offsets[e] = off;
      if (tot[r] > 0 && a.active) a.active[act] = e;
      if (e == E - 1) {
        a.offsets[E] = off + tot[r];
        if (a.nactive) *a.nactive = act + (tot[r] > 0);
      }
    }
    act += tot[r] > 0;
    off += tot[r];
  }

  // pass 1: per-warp counts of this CTA's pairs; warp w owns a contiguous share
  int clo, chi;
  cta_pairs(a, c, clo, chi);
  const int n = chi - clo;
  const int lo = clo + (int)((long long)warp * n / BK_PLACE_WARPS);
  const int hi = clo + (int)((long long)(warp + 1) * n / BK_PLACE_WARPS);
  for (int p0 = lo + lane; p0 < hi; p0 += 128) {
    int ev[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) ev[u] = p0 + 32 * u < hi ? a.idx[p0 + 32 * u] : -1;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if ((unsigned)ev[u] < (unsigned)E) atomicAdd(&hist[warp * E + ev[u]], 1);
  }
  __syncthreads();
  // running start of each (warp, expert) run: CTA base, then the warps before
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    if (e >= E) continue;
    int s = base[r];
    for (int w = 0; w < BK_PLACE_WARPS; ++w) {
      const int cw = hist[w * E + e];
      hist[w * E + e] = s;
      s += cw;
    }
  }
  __syncthreads();
  // pass 2: place this warp's pairs in pair order, 32 at a time; the expert
  // ids of the next batches are loaded ahead
  int nxt[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) nxt[u] = lo + lane + 32 * u < hi ? a.idx[lo + lane + 32 * u] : 0;
  for (int p0 = lo; p0 < hi; p0 += 128) {
    int cur[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      cur[u] = nxt[u];
      const int q = p0 + 128 + lane + 32 * u;
      nxt[u] = q < hi ? a.idx[q] : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + 32 * u + lane;
      if (p0 + 32 * u >= hi) break;           // warp-uniform
      const bool valid = p < hi && (unsigned)cur[u] < (unsigned)E;
      const int e = valid ? cur[u] : -1 - lane;   // distinct dummy keys for the tail
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int pos = 0;
      if (valid) pos = hist[warp * E + e] + rank;
      __syncwarp();
      if (valid && rank == 0) hist[warp * E + e] += __popc(peers);
      __syncwarp();
      if (valid) {
        a.perm[pos] = p;
        if (a.ptok) a.ptok[pos] = p / a.k;
        if (a.pgate) a.pgate[pos] = a.gate[p];
      }
    }
  }
}

int bucket_ctas(int T) {
  const int per = std::max(BK_MIN_TOKENS, (T + BK_MAX_CTAS - 1) / BK_MAX_CTAS);
  return std::max(1, (T + per - 1) / per);
}

}  // namespace

size_t bucket_ws_bytes(int T, int k, int E) {
  (void)k;
  const size_t C = (size_t)bucket_ctas(T);
  return ((C * E * sizeof(int32_t) + 255) & ~(size_t)255) + ((C * sizeof(int32_t) + 255) & ~(size_t)255);
}

bool bucket_supported(int T, int k, int E) {
  return E >= 1 && E <= BK_MAX_E && (long long)T * k <= (1LL << 30) &&
         (size_t)BK_PLACE_WARPS * E * sizeof(int) <= max_smem_optin();
}

qmoe_status bucket_launch(const int32_t *idx, const float *gate, int T, int k, int E, void *ws, int32_t *offsets,
                          int32_t *perm, int32_t *ptok, float *pgate, int32_t *active, int32_t *nactive,
                          bool check_dup, int32_t *status, cudaStream_t s) {
  const int C = bucket_ctas(T);
  int32_t *cnt = static_cast<int32_t *>(ws);
  int32_t *flag = reinterpret_cast<int32_t *>(static_cast<char *>(ws) +
                                              (((size_t)C * E * sizeof(int32_t) + 255) & ~(size_t)255));
  BucketArgs a{idx, gate, T, k, E, C, cnt, flag, offsets, perm, ptok, pgate, active, nactive,
               check_dup ? 1 : 0, status};
  const size_t smem = (size_t)BK_PLACE_WARPS * E * sizeof(int);
  if (cudaFuncSetAttribute(bk_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMOE_ERR_CUDA;
  bk_count_kernel<<<C, BK_COUNT_THREADS, E * sizeof(int), s>>>(a);
  bk_place_kernel<<<C, BK_PLACE_THREADS, smem, s>>>(a);
  note_launch(2);
  return cuda_status(cudaGetLastError());
}

}  // namespace qmoe

using namespace qmoe;

extern "C" size_t qmoe_bucket_workspace_bytes(int T, int k, int E) {
  if (T < 1 || k < 1 || E < 1) return 0;
  return bucket_ws_bytes(T, k, E);
}

extern "C" qmoe_status qmoe_bucket(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm,
                                   int32_t *active, int32_t *nactive, void *workspace, size_t workspace_bytes,
                                   int32_t *dev_status, qmoe_stream_t stream) {
  if (!idx || !offsets || !perm || !workspace || !dev_status) return QMOE_ERR_INVALID_ARG;
  if (T < 1 || k < 1 || E < 1) return QMOE_ERR_INVALID_ARG;
  if (E > BK_MAX_E || (long long)T * k > (1LL << 30)) return QMOE_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(offsets) |
                       reinterpret_cast<uintptr_t>(perm) | reinterpret_cast<uintptr_t>(active) |
                       reinterpret_cast<uintptr_t>(nactive) | reinterpret_cast<uintptr_t>(dev_status);
  if (al & 3) return QMOE_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return QMOE_ERR_INVALID_ARG;
  if (workspace_bytes < bucket_ws_bytes(T, k, E)) return QMOE_ERR_WORKSPACE;
  if (!bucket_supported(T, k, E)) return QMOE_ERR_UNSUPPORTED;
  return bucket_launch(idx, nullptr, T, k, E, workspace, offsets, perm, nullptr, nullptr, active, nactive, false,
                       dev_status, (cudaStream_t)stream);
}
