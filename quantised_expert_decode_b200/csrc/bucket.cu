// Token -> expert bucketing for prefill chunks: a stable counting sort of the
// (token, slot) pairs by expert. Pairs are numbered p = t*k + j; the sorted
// order is (expert, t, j), so the permutation is unique and reproducible.
#include "common.cuh"

namespace qmoe {
namespace {

constexpr int BK_THREADS = 1024;
constexpr int BK_WARPS = BK_THREADS / 32;
constexpr int BK_MAX_E = 1024;   // 32 per-warp histograms of E counters fit shared memory

struct BucketArgs {
  const int32_t *idx;   // [P]
  const float *gate;    // [P] or null
  int P, k, E;
  int32_t *offsets;     // [E + 1]
  int32_t *perm;        // [P] sorted position -> pair id
  int32_t *ptok;        // [P] or null: token of each sorted pair
  float *pgate;         // [P] or null: gate of each sorted pair
  int32_t *active;      // [E] or null: experts with at least one pair, ascending
  int32_t *nactive;     // [1] or null
  int check_dup;        // report an expert repeated within one token's route
  int32_t *status;
};

// One CTA. Warp w owns pairs [w*P/32, (w+1)*P/32): it counts them per expert
// (pass 1); a prefix over (expert, warp) gives each warp its first sorted
// position per expert; pass 2 places the warp's pairs in pair order, so equal
// experts keep pair order. Thread i owns experts 2i and 2i+1 in the scans.
__global__ void __launch_bounds__(BK_THREADS, 1) bucket_kernel(BucketArgs a) {
  extern __shared__ int hist[];   // [BK_WARPS][E]: counts, then running positions
  __shared__ int bad;
  __shared__ int wtot[3][BK_WARPS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E;
  for (int i = tid; i < BK_WARPS * E; i += BK_THREADS) hist[i] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  const int lo = (int)((long long)warp * a.P / BK_WARPS), hi = (int)((long long)(warp + 1) * a.P / BK_WARPS);
  // four pairs per lane per step, loads issued before use
  for (int p0 = lo + lane; p0 < hi; p0 += 128) {
    int ev[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) ev[u] = p0 + 32 * u < hi ? a.idx[p0 + 32 * u] : 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + 32 * u;
      if (p >= hi) continue;
      const int e = ev[u];
      if (e < 0 || e >= E) {
        bad = 1;
        continue;
      }
      if (a.check_dup) {
        const int j = p % a.k;
        for (int j2 = 0; j2 < j; ++j2)
          if (a.idx[p - j + j2] == e) bad = 2;
      }
      atomicAdd(&hist[warp * E + e], 1);
    }
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(a.status, bad == 1 ? DEV_BAD_INDEX : DEV_DUP_INDEX);
    return;
  }
  // column prefix over warps for this thread's two experts
  int tot[2] = {0, 0};
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    if (e < E) {
      int s = 0;
      for (int w = 0; w < BK_WARPS; ++w) {
        const int c = hist[w * E + e];
        hist[w * E + e] = s;
        s += c;
      }
      tot[r] = s;
    }
  }
  // block-wide exclusive scans of pair counts and active flags
  const int v = tot[0] + tot[1];
  const int f = (tot[0] > 0) + (tot[1] > 0);
  int iv = v, ifl = f, dummy = 0;
  warp_scan3(iv, ifl, dummy);
  if (lane == 31) {
    wtot[0][warp] = iv;
    wtot[1][warp] = ifl;
  }
  __syncthreads();
  if (warp == 0) {
    int s0 = wtot[0][lane], s1 = wtot[1][lane], s2 = 0;
    int i0 = s0, i1 = s1;
    warp_scan3(i0, i1, s2);
    wtot[0][lane] = i0 - s0;
    wtot[1][lane] = i1 - s1;
  }
  __syncthreads();
  int off = wtot[0][warp] + iv - v;
  int act = wtot[1][warp] + ifl - f;
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    if (e < E) {
      a.offsets[e] = off;
      for (int w = 0; w < BK_WARPS; ++w) hist[w * E + e] += off;
      if (tot[r] > 0 && a.active) a.active[act] = e;
      act += tot[r] > 0;
      off += tot[r];
      if (e == E - 1) {
        a.offsets[E] = off;
        if (a.nactive) *a.nactive = act;
      }
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
      const bool valid = p < hi;
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

}  // namespace

size_t bucket_smem_bytes(int E) { return (size_t)BK_WARPS * E * sizeof(int); }

bool bucket_supported(int T, int k, int E) {
  return E >= 1 && E <= BK_MAX_E && (long long)T * k <= (1LL << 30) && bucket_smem_bytes(E) <= max_smem_optin();
}

qmoe_status bucket_launch(const int32_t *idx, const float *gate, int T, int k, int E, int32_t *offsets, int32_t *perm,
                          int32_t *ptok, float *pgate, int32_t *active, int32_t *nactive, bool check_dup,
                          int32_t *status, cudaStream_t s) {
  BucketArgs a{idx, gate, T * k, k, E, offsets, perm, ptok, pgate, active, nactive, check_dup ? 1 : 0, status};
  const size_t smem = bucket_smem_bytes(E);
  if (cudaFuncSetAttribute(bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMOE_ERR_CUDA;
  bucket_kernel<<<1, BK_THREADS, smem, s>>>(a);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace qmoe

using namespace qmoe;

extern "C" qmoe_status qmoe_bucket(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm,
                                   int32_t *active, int32_t *nactive, int32_t *dev_status, qmoe_stream_t stream) {
  if (!idx || !offsets || !perm || !dev_status) return QMOE_ERR_INVALID_ARG;
  if (T < 1 || k < 1 || E < 1) return QMOE_ERR_INVALID_ARG;
  if (E > BK_MAX_E || (long long)T * k > (1LL << 30)) return QMOE_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(offsets) |
                       reinterpret_cast<uintptr_t>(perm) | reinterpret_cast<uintptr_t>(active) |
                       reinterpret_cast<uintptr_t>(nactive) | reinterpret_cast<uintptr_t>(dev_status);
  if (al & 3) return QMOE_ERR_INVALID_ARG;
  if (!bucket_supported(T, k, E)) return QMOE_ERR_UNSUPPORTED;
  return bucket_launch(idx, nullptr, T, k, E, offsets, perm, nullptr, nullptr, active, nactive, false,
                       dev_status, (cudaStream_t)stream);
}
