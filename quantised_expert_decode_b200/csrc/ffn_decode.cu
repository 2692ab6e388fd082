// Routed expert FFN + gate-weighted combine for decode / verify batches (T <= 8).
//
// One grid of one CTA per SM (all resident), three phases separated by grid barriers:
//   phase 1  gate and up projections: items are (expert, gate|up, 16-row tile)
//            over K = H; results a_g, a_u go to the workspace.
//   phase 2  down projection: items are (expert, 32-row tile) over K = I on
//            h = silu(a_g) * a_u; each result is scaled by its gate and stored
//            per (token, slot).
//   phase 3  y[t] = sum over slots j (in slot order) of the phase-2 results.
// Weights stream HBM -> shared memory through bulk asynchronous copies issued by
// one producer thread into a ring of slots (mbarrier full/empty pairs); the
// copies of phase-2 tiles start as soon as ring slots free up, so they overlap
// phase 1 and the first grid barrier.
//
// The contraction itself (limb quantisation, integer MMA tiles) lives in
// decode_tile.cuh, shared with the fused layer-stack kernel.
#include <cuda_fp16.h>

#include "common.cuh"
#include "decode_canon.cuh"
#include "decode_tile.cuh"
#include "layout.cuh"

namespace qmoe {
namespace {
using namespace tile;

constexpr int NCW = 8;                     // consumer warps
constexpr int FD_THREADS = 32 * (NCW + 1); // + one producer warp
constexpr int FD_MAXT = 8;
constexpr int FD_MAXK = 16;
constexpr int FD_MAXP = FD_MAXT * FD_MAXK; // (token, slot) pairs
constexpr int FD_MAXE = 1024;              // experts a layer
static_assert(FD_MAXP % 32 == 0 && FD_MAXT <= 8, "plan layout: 32-pair rows, one byte of tokens an expert");
constexpr int CONSUMER_BAR = 1;            // named barrier id for the consumer warps
struct Plan {
  int err;
  int abort;
  int U;
  int ue[FD_MAXP];
  int nt[FD_MAXP];
  int pbase[FD_MAXP + 1];
  int ptok[FD_MAXP];
  int pslot[FD_MAXP];
  float pgate[FD_MAXP];
  int cw[FD_MAXP + 1];      // exclusive prefix of tile_cost(nt[u])
  unsigned tm[FD_MAXE / 4]; // per expert, one byte: the tokens (bits) routed to it
  int wbase[32];            // experts in the bitmap words before word w
  unsigned bm[32];          // bitmap of the routed experts
  int vids[NCW][FD_MAXT];   // per consumer warp: limb-region vectors of the current item
  int lo1, hi1, lo2, hi2;   // this CTA's gate/up and down item ranges
};

// Relative cost of a tile whose expert serves n tokens. With a warp per SM
// sub-partition or more the tiles are issue-bound, so the cost follows the
// instructions of the tile-dot variant for n vectors (NP = 1, 2, 4, 8: about
// 15, 23, 46 and 90 a block and lane).
__device__ __forceinline__ int tile_cost(int n) { return n <= 1 ? 2 : n <= 2 ? 3 : n <= 4 ? 6 : 12; }

__device__ __forceinline__ int warp_excl_scan(int v, int &total) {
  const int lane = threadIdx.x & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  total = __shfl_sync(0xffffffffu, incl, 31);
  return incl - v;
}

// One warp. Items are numbered expert by expert, per_expert items an expert,
// each at its expert's tile cost (cost prefix cw). For each of the NT targets
// returns the first item whose starting cost is at least that target
// (U * per_expert if none). Expert u holds that item when it is the first with
// target <= acc_u + (per_expert - 1) w_u, acc_u = per_expert cw[u]: the item is
// then u's first if target <= acc_u, else the ceil((target - acc_u) / w_u)-th.
// All targets are resolved in one pass over the experts, in 32-bit arithmetic
// (the caller checks the costs fit).
template <int NT>
__device__ __forceinline__ void items_at_costs(const Plan *pl, int U, int per_expert, const int (&target)[NT],
                                               int (&item)[NT]) {
  const int lane = threadIdx.x & 31;
  bool done[NT];
#pragma unroll
  for (int q = 0; q < NT; ++q) {
    done[q] = false;
    item[q] = U * per_expert;
  }
  for (int u0 = 0; u0 < U; u0 += 32) {
    const int u = u0 + lane;
    int acc = 0, w = 1;
    if (u < U) {
      w = tile_cost(pl->nt[u]);
      acc = per_expert * pl->cw[u];
    }
#pragma unroll
    for (int q = 0; q < NT; ++q) {
      const unsigned b = __ballot_sync(0xffffffffu, u < U && target[q] <= acc + (per_expert - 1) * w);
      if (!done[q] && b) {
        const int src = __ffs(b) - 1;
        const int acc0 = __shfl_sync(0xffffffffu, acc, src);
        const int w0 = __shfl_sync(0xffffffffu, w, src);
        const int ui = u0 + src;
        item[q] = target[q] <= acc0 ? ui * per_expert : ui * per_expert + (target[q] - acc0 + w0 - 1) / w0;
        done[q] = true;
      }
    }
  }
}

// Route table -> unique experts (ascending), their tokens (ascending) and
// slots, and the tile-cost prefix; one warp, every step spread over the lanes.
__device__ void build_plan(const int32_t *idx, const float *gate, int T, int k, int E, int32_t *status, Plan *pl) {
  const int lane = threadIdx.x & 31;
  const int P = T * k;
  for (int w = lane; w < FD_MAXE / 4; w += 32) pl->tm[w] = 0u;
  int pe[FD_MAXP / 32];
  float pg[FD_MAXP / 32];
#pragma unroll 1
  for (int i = 0; i < FD_MAXP / 32; ++i) {
    const int p = lane + 32 * i;
    pe[i] = p < P ? idx[p] : 0;
    pg[i] = p < P ? gate[p] : 0.0f;
  }
  __syncwarp();
  int bad = 0;
#pragma unroll 1
  for (int i = 0; i < FD_MAXP / 32; ++i) {
    const int p = lane + 32 * i;
    if (p >= P) continue;
    const int e = pe[i];
    if (e < 0 || e >= E) {
      bad = DEV_BAD_INDEX;
      continue;
    }
    const unsigned bit = 1u << ((e & 3) * 8 + p / k);
    if (atomicOr(&pl->tm[e >> 2], bit) & bit) bad = DEV_DUP_INDEX;   // the token names e twice
  }
  const unsigned badmask = __ballot_sync(0xffffffffu, bad != 0);
  if (badmask) {
    const int code = __shfl_sync(0xffffffffu, bad, __ffs(badmask) - 1);
    if (lane == 0) {
      pl->err = code;
      set_status(status, code);
    }
    __syncwarp();
    return;
  }
  __syncwarp();
  // bitmap word `lane`: experts 32 lane .. 32 lane + 31
  unsigned word = 0u;
#pragma unroll 1
  for (int q = 0; q < 8; ++q) {
    const unsigned m = pl->tm[lane * 8 + q];
#pragma unroll 1
    for (int b = 0; b < 4; ++b)
      if ((m >> (8 * b)) & 0xffu) word |= 1u << (4 * q + b);
  }
  int U;
  const int wb = warp_excl_scan(__popc(word), U);
  pl->bm[lane] = word;
  pl->wbase[lane] = wb;
  for (unsigned w2 = word, r = wb; w2; w2 &= w2 - 1u, ++r) {
    const int e = lane * 32 + __ffs(w2) - 1;
    pl->ue[r] = e;
    pl->nt[r] = __popc((pl->tm[e >> 2] >> ((e & 3) * 8)) & 0xffu);
  }
  __syncwarp();
  // token and cost prefixes over the unique experts (4 a lane, in order)
  int nt4[FD_MAXP / 32], c4[FD_MAXP / 32], ntl = 0, cl = 0;
#pragma unroll 1
  for (int i = 0; i < FD_MAXP / 32; ++i) {
    const int u = lane * (FD_MAXP / 32) + i;
    nt4[i] = u < U ? pl->nt[u] : 0;
    c4[i] = u < U ? tile_cost(nt4[i]) : 0;
    ntl += nt4[i];
    cl += c4[i];
  }
  int ntot, ctot;
  int nb = warp_excl_scan(ntl, ntot), cb = warp_excl_scan(cl, ctot);
#pragma unroll 1
  for (int i = 0; i < FD_MAXP / 32; ++i) {
    const int u = lane * (FD_MAXP / 32) + i;
    if (u < U) {
      pl->pbase[u] = nb;
      pl->cw[u] = cb;
    }
    nb += nt4[i];
    cb += c4[i];
  }
  if (lane == 0) {
    pl->pbase[U] = ntot;
    pl->cw[U] = ctot;
    pl->U = U;
    pl->err = 0;
    pl->abort = 0;
  }
  __syncwarp();
  // each pair's place among its expert's tokens (token order)
#pragma unroll 1
  for (int i = 0; i < FD_MAXP / 32; ++i) {
    const int p = lane + 32 * i;
    if (p < P) {
      const int e = pe[i], t = p / k;
      const int u = pl->wbase[e >> 5] + __popc(pl->bm[e >> 5] & ((1u << (e & 31)) - 1u));
      const unsigned toks = (pl->tm[e >> 2] >> ((e & 3) * 8)) & 0xffu;
      const int q = pl->pbase[u] + __popc(toks & ((1u << t) - 1u));
      pl->ptok[q] = t;
      pl->pslot[q] = p % k;
      pl->pgate[q] = pg[i];
    }
  }
  __syncwarp();
}

struct FfnArgs {
  const uint8_t *gu;
  const uint8_t *dn;
  const float *x;
  const int32_t *idx;
  const float *gate;
  float *y;
  float *abuf;    // [P][2][I]
  float *part;    // [T][k][H]
  uint8_t *xlimbs;  // [T][H/32][LIMB_REC] limbs of x, quantised once across the grid
  float2 *xlsc;     // [T][H/32] their block scales
  unsigned *bar;  // grid barrier counter
  int32_t *status;
  int T, k, E, H, I;
  int slot_bytes, nslots;
  int ncons;       // consumer warps that take ring items; nslots is a multiple of it
  int limb_bytes;  // activation-limb region
  int lsc_count;   // float2 entries of the limb-scale table
};

// Shared-memory carve-up (byte offsets from the dynamic base), used by host and device.
struct SmemLayout {
  size_t bars, plan, limbs, lsc, total;
};
__host__ __device__ inline SmemLayout smem_layout(int nslots, int slot_bytes, int limb_bytes, int lsc_count) {
  SmemLayout o;
  o.bars = (size_t)nslots * slot_bytes;                       // slot_bytes is a multiple of 128
  o.plan = (o.bars + (size_t)nslots * 16 + 8 + 15) & ~(size_t)15;   // full, empty per slot; the x-limb barrier
  o.limbs = (o.plan + sizeof(Plan) + 127) & ~(size_t)127;
  o.lsc = (o.limbs + (size_t)limb_bytes + 15) & ~(size_t)15;
  o.total = o.lsc + (size_t)lsc_count * 8;
  return o;
}

template <int BITS>
__global__ void __launch_bounds__(FD_THREADS, 1) ffn_decode_kernel(FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.nslots;
  const SmemLayout lay = smem_layout(S, a.slot_bytes, a.limb_bytes, a.lsc_count);
  uint8_t *ring = smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.bars);
  uint64_t *empty = full + S;
  uint64_t *xbar = empty + S;
  Plan *pl = reinterpret_cast<Plan *>(smem + lay.plan);
  uint8_t *limbs = smem + lay.limbs;
  float2 *lsc = reinterpret_cast<float2 *>(smem + lay.lsc);

  const int H = a.H, I = a.I, k = a.k;
  const int nblkH = H / 32, nblkI = I / 32;
  const int I16 = I / 16, H16 = H / 16;
  const int tgu = tile_bytes(BITS, H), tdn = tile_bytes(BITS, I);
  const unsigned G = gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(xbar, 1);
    fence_mbar_init();
  }
  // Everything above overlaps the previous kernel; idx, gate and x are its outputs.
  pdl_wait();
  if (warp == 0) {
    build_plan(a.idx, a.gate, a.T, a.k, a.E, a.status, pl);
    // split both phases' items over the CTAs by cost, not by count: a tile
    // shared by 8 tokens costs several times a single-token tile
    if (!pl->err) {
      // total costs: at most 128 experts x 12 x (2 I / 16 or H / 16) items,
      // times G < 2^31 for the shapes the launch admits (checked there)
      const int U = pl->U;
      const long long W = pl->cw[U], W1 = W * 2 * I16, W2 = W * H16;
      const int t1[2] = {(int)(W1 * blockIdx.x / G), (int)(W1 * (blockIdx.x + 1) / G)};
      const int t2[2] = {(int)(W2 * blockIdx.x / G), (int)(W2 * (blockIdx.x + 1) / G)};
      int r1[2], r2[2];
      items_at_costs<2>(pl, U, 2 * I16, t1, r1);
      items_at_costs<2>(pl, U, H16, t2, r2);
      if (lane == 0) {
        pl->lo1 = r1[0];
        pl->hi1 = r1[1];
        pl->lo2 = r2[0];
        pl->hi2 = r2[1];
      }
    }
  }
  __syncthreads();
  if (pl->err) return;

  const int lo1 = pl->lo1, hi1 = pl->hi1, lo2 = pl->lo2, hi2 = pl->hi2;
  const int n1 = hi1 - lo1, ntot = n1 + (hi2 - lo2);

  if (warp == NCW) {
    // ------------------------------------------------------------ producer --
    // Lane s issues every copy into ring slot s, in item order (item n goes to
    // slot n % S). One thread's bulk copies are serviced one after another, so
    // several issuers keep more bytes in flight; keeping each slot's copies on
    // one lane and in order means each wait below is at most one phase behind
    // its barrier, which is what a parity wait can tell apart.
    int my_last = -1;
    bool aborted = false;
    const uint64_t pol = l2_evict_first();
    for (int n = lane; lane < S && n < ntot; n += S) {
      const int s = n % S, it = n / S;
      if (n >= S) {
        const long long dl = clock64() + WAIT_BUDGET_CYCLES;
        while (!mbar_try_wait(&empty[s], (uint32_t)((it - 1) & 1))) {
          if (*(volatile int *)&pl->abort || clock64() > dl) {
            aborted = true;
            break;
          }
        }
        if (aborted) break;
      }
      const uint8_t *src;
      uint32_t bytes;
      if (n < n1) {
        const int i = lo1 + n;
        const int u = i / (2 * I16), m = (i / I16) & 1, r = i % I16;
        src = a.gu + (((size_t)pl->ue[u] * 2 + m) * I16 + r) * (size_t)tgu;
        bytes = (uint32_t)tgu;
      } else {
        const int i = lo2 + (n - n1);
        const int u = i / H16, r = i % H16;
        src = a.dn + ((size_t)pl->ue[u] * H16 + r) * (size_t)tdn;
        bytes = (uint32_t)tdn;
      }
      mbar_arrive_expect_tx(&full[s], bytes);
      bulk_g2s_hint(ring + (size_t)s * a.slot_bytes, src, bytes, &full[s], pol);
      my_last = n;
    }
    // never leave with copies in flight: wait for this lane's copies whose slot
    // was not reused (reuse implies the copy was consumed)
    const long long dl = clock64() + WAIT_BUDGET_CYCLES;
    for (int n = lane; n <= my_last; n += S) {
      if (!aborted && n + S < ntot) continue;
      while (!mbar_try_wait(&full[n % S], (uint32_t)((n / S) & 1)))
        if (clock64() > dl) break;
    }
    pdl_launch_dependents();
    return;
  }

  // ---------------------------------------------------------------- consumers --
  const int nth = NCW * 32;
  // Grid barrier of the consumer threads (the producer never joins one).
  auto grid_sync = [&]() {
    named_barrier_sync(CONSUMER_BAR, nth);
    if (tid == 0) {
      if (!*(volatile int *)&pl->abort && !grid_barrier_one_thread(a.bar, G)) {
        set_status(a.status, DEV_TIMEOUT);
        *(volatile int *)&pl->abort = 1;
      }
      __threadfence();
    }
    named_barrier_sync(CONSUMER_BAR, nth);
  };

  // Activation limbs of the T tokens: the 128-element chunks are spread over
  // the grid (chunk task of CTA task % G), quantised once into the workspace,
  // and after a grid barrier every CTA copies all of them into shared memory.
  {
    const int nch = H / 128, ntask = a.T * nch;
    for (int task = blockIdx.x + G * warp; task < ntask; task += G * NCW) {
      const int t = task / nch, c = task % nch;
      const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.x + (size_t)t * H + c * 128) + lane);
      quant_chunk(v, a.xlimbs + (size_t)t * nblkH * LIMB_REC, a.xlsc + (size_t)t * nblkH, c, lane);
    }
  }
  grid_sync();
  {
    const uint32_t lb = (uint32_t)(a.T * nblkH * LIMB_REC), sb = (uint32_t)(a.T * nblkH * 8);
    if (tid == 0) {
      fence_proxy_async();   // the limbs were written with ordinary stores
      mbar_arrive_expect_tx(xbar, lb + sb);
      bulk_g2s(limbs, a.xlimbs, lb, xbar);
      bulk_g2s(lsc, a.xlsc, sb, xbar);
    }
    if (!mbar_wait(xbar, 0u, clock64() + WAIT_BUDGET_CYCLES)) {
      set_status(a.status, DEV_TIMEOUT);
      *(volatile int *)&pl->abort = 1;
    }
  }
  named_barrier_sync(CONSUMER_BAR, nth);

  // Waits for ring item n. Item n goes to slot n % S and to consumer warp
  // n % NA, and S is a multiple of NA, so every slot has one consumer warp,
  // which takes the slot's phases in order: when it waits for item n it has
  // already consumed item n - S of the same slot, so the slot's barrier is in
  // the phase of item n and the parity wait is exact.
  const int NA = a.ncons;
  auto wait_full = [&](int n) -> bool {
    const long long dl = clock64() + WAIT_BUDGET_CYCLES;
    const uint32_t par = (uint32_t)((n / S) & 1);
    while (!mbar_try_wait(&full[n % S], par)) {
      if (*(volatile int *)&pl->abort) return false;
      if (clock64() > dl) {
        set_status(a.status, DEV_TIMEOUT);
        *(volatile int *)&pl->abort = 1;
        return false;
      }
    }
    return true;
  };
  auto release = [&](int n) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[n % S]);
  };
  const int g = lane >> 2, t = lane & 3;

  // phase 1: gate / up
  for (int n = warp; warp < NA && n < n1; n += NA) {
    if (!wait_full(n)) break;
    const int i = lo1 + n;
    const int u = i / (2 * I16), m = (i / I16) & 1, r = i % I16;
    const uint8_t *tile = ring + (size_t)(n % S) * a.slot_bytes;
    const int nu = pl->nt[u], pb = pl->pbase[u];
    Acc acc;
    const int np = dispatch_dot<BITS>(tile, nblkH, limbs, lsc, &pl->ptok[pb], nu, acc);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int tau = owner(np, t, q);
      if (tau >= 0 && tau < nu) {
        float *dst = a.abuf + ((size_t)(pb + tau) * 2 + m) * I + r * 16;
        dst[g] = acc.r0[q];
        dst[g + 8] = acc.r1[q];
      }
    }
    release(n);
  }

  // grid barrier 1: every a_g / a_u is written
  grid_sync();
  // all CTAs of this grid are resident now; the next kernel may start its prologue
  pdl_launch_dependents();
  bool ok = !*(volatile int *)&pl->abort;

  // phase 2: down projection, one expert chunk at a time
  const int hmaxp = a.limb_bytes / (I * 3);
  int item = lo2;
  while (ok && item < hi2) {
    const int u0 = item / H16;
    const int ulast = (hi2 - 1) / H16;
    int u1 = u0, pairs = 0;
    while (u1 <= ulast && pairs + pl->nt[u1] <= hmaxp) {
      pairs += pl->nt[u1];
      ++u1;
    }
    if (u1 == u0) {  // cannot happen: hmaxp >= FD_MAXT >= any expert's token count
      set_status(a.status, DEV_BAD_INDEX);
      *(volatile int *)&pl->abort = 1;
      break;
    }
    const int pb0 = pl->pbase[u0];
    {
      const int nch = I / 128;
      const float *abuf = a.abuf;
      quant_tasks<NCW, 8>(pairs * nch, nch, nblkI, limbs, lsc, warp, lane, [&](int lv, int c) {
        const float *ab = abuf + (size_t)(pb0 + lv) * 2 * I + c * 128;
        float4 gv = __ldcg(reinterpret_cast<const float4 *>(ab) + lane);
        float4 uv = __ldcg(reinterpret_cast<const float4 *>(ab + I) + lane);
        return make_float4(canon::hval(gv.x, uv.x), canon::hval(gv.y, uv.y), canon::hval(gv.z, uv.z),
                           canon::hval(gv.w, uv.w));
      });
    }
    named_barrier_sync(CONSUMER_BAR, nth);
    const int item_end = min(hi2, u1 * H16);
    for (int it2 = item; it2 < item_end; ++it2) {
      const int n = n1 + (it2 - lo2);
      if (n % NA != warp) continue;
      if (!wait_full(n)) break;
      const int u = it2 / H16, r = it2 % H16;
      const int nu = pl->nt[u], pb = pl->pbase[u];
      int *vid = pl->vids[warp];
      if (lane < FD_MAXT) vid[lane] = pb - pb0 + lane;
      __syncwarp();
      const uint8_t *tile = ring + (size_t)(n % S) * a.slot_bytes;
      Acc acc;
      const int np = dispatch_dot<BITS>(tile, nblkI, limbs, lsc, vid, nu, acc);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int tau = owner(np, t, q);
        if (tau >= 0 && tau < nu) {
          const int p = pb + tau;
          const float gw = pl->pgate[p];
          float *dst = a.part + ((size_t)pl->ptok[p] * k + pl->pslot[p]) * H + r * 16;
          dst[g] = __fmul_rn(gw, acc.r0[q]);
          dst[g + 8] = __fmul_rn(gw, acc.r1[q]);
        }
      }
      release(n);
    }
    named_barrier_sync(CONSUMER_BAR, nth);
    ok = !*(volatile int *)&pl->abort;
    item = item_end;
  }

  // grid barrier 2: every gated expert output is written
  grid_sync();
  if (*(volatile int *)&pl->abort) return;

  // phase 3: y[t] = sum_j part[t][j] in slot order
  const int H4 = H / 4;
  const float4 *p4 = reinterpret_cast<const float4 *>(a.part);
  float4 *y4 = reinterpret_cast<float4 *>(a.y);
  for (int o = blockIdx.x * nth + tid; o < a.T * H4; o += G * nth) {
    const int tt = o / H4, h = o % H4;
    float4 v[FD_MAXK];
#pragma unroll
    for (int j = 0; j < FD_MAXK; ++j)
      if (j < k) v[j] = __ldcg(p4 + ((size_t)tt * k + j) * H4 + h);
    // slot order, one rounding per add: the combine of decode_canon.cuh
    // (gate * result was rounded once in phase 2)
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < FD_MAXK; ++j)
      if (j < k) {
        sum.x = __fadd_rn(sum.x, v[j].x); sum.y = __fadd_rn(sum.y, v[j].y);
        sum.z = __fadd_rn(sum.z, v[j].z); sum.w = __fadd_rn(sum.w, v[j].w);
      }
    y4[o] = sum;
  }
}

size_t ws_bar_bytes() { return 256; }
size_t ws_abuf_bytes(int T, int k, int I) { return (((size_t)T * k * 2 * I * 4) + 255) & ~(size_t)255; }
size_t ws_part_bytes(int T, int k, int H) { return (((size_t)T * k * H * 4) + 255) & ~(size_t)255; }
size_t ws_xlimb_bytes(int T, int H) { return (((size_t)T * (H / 32) * LIMB_REC) + 255) & ~(size_t)255; }
size_t ws_xlsc_bytes(int T, int H) { return (((size_t)T * (H / 32) * 8) + 255) & ~(size_t)255; }

}  // namespace
}  // namespace qmoe

namespace qmoe {
qmoe_status ffn_decode_launch(const qmoe_experts *ex, const float *x, int T, const int32_t *idx, const float *gate,
                              int k, float *y, void *ws, size_t ws_bytes, int32_t *status, cudaStream_t s,
                              bool cooperative);
}

using namespace qmoe;

extern "C" size_t qmoe_decode_workspace_bytes(int T, int k, int H, int I) {
  if (T < 1 || k < 1 || H < 1 || I < 1) return 0;
  return ws_bar_bytes() + ws_abuf_bytes(T, k, I) + ws_part_bytes(T, k, H) + ws_xlimb_bytes(T, H) + ws_xlsc_bytes(T, H);
}

qmoe_status qmoe::ffn_decode_launch(const qmoe_experts *ex, const float *x, int T, const int32_t *idx,
                                    const float *gate, int k, float *y, void *workspace, size_t workspace_bytes,
                                    int32_t *dev_status, cudaStream_t stream, bool cooperative) {
  if (!ex || !x || !idx || !gate || !y || !workspace || !dev_status) return QMOE_ERR_INVALID_ARG;
  if (!ex->gate_up || !ex->down) return QMOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace) || !aligned16(ex->gate_up) || !aligned16(ex->down) ||
      (reinterpret_cast<uintptr_t>(idx) & 3) || (reinterpret_cast<uintptr_t>(gate) & 3))
    return QMOE_ERR_INVALID_ARG;
  if (ex->fmt != QMOE_Q2 && ex->fmt != QMOE_Q4) return QMOE_ERR_GEOMETRY;
  if (ex->E < 1 || ex->H < 128 || ex->I < 128 || ex->H % 128 || ex->I % 128 || ex->E > 1024) return QMOE_ERR_GEOMETRY;
  if (ex->gate_up_bytes != qmoe_packed_bytes(ex->fmt, QMOE_GATE_UP, ex->E, ex->H, ex->I) ||
      ex->down_bytes != qmoe_packed_bytes(ex->fmt, QMOE_DOWN, ex->E, ex->H, ex->I))
    return QMOE_ERR_GEOMETRY;
  if (T < 1 || T > FD_MAXT || k < 1 || k > FD_MAXK || k > ex->E) return QMOE_ERR_UNSUPPORTED;
  // the cost split runs in 32-bit integers: at most 128 experts x cost 12 x items
  // an expert, times the grid
  if ((long long)FD_MAXP * 12 * ((2 * ex->I > ex->H ? 2 * ex->I : ex->H) / 16) * num_sms() >= (1LL << 31))
    return QMOE_ERR_UNSUPPORTED;
  if (workspace_bytes < qmoe_decode_workspace_bytes(T, k, ex->H, ex->I)) return QMOE_ERR_WORKSPACE;

  const int bits = ex->fmt, H = ex->H, I = ex->I;
  FfnArgs a{};
  a.gu = static_cast<const uint8_t *>(ex->gate_up);
  a.dn = static_cast<const uint8_t *>(ex->down);
  a.x = x;
  a.idx = idx;
  a.gate = gate;
  a.y = y;
  char *ws = static_cast<char *>(workspace);
  a.bar = reinterpret_cast<unsigned *>(ws);
  a.abuf = reinterpret_cast<float *>(ws + ws_bar_bytes());
  a.part = reinterpret_cast<float *>(ws + ws_bar_bytes() + ws_abuf_bytes(T, k, I));
  a.xlimbs = reinterpret_cast<uint8_t *>(ws + ws_bar_bytes() + ws_abuf_bytes(T, k, I) + ws_part_bytes(T, k, ex->H));
  a.xlsc = reinterpret_cast<float2 *>(a.xlimbs + ws_xlimb_bytes(T, ex->H));
  a.status = dev_status;
  a.T = T; a.k = k; a.E = ex->E; a.H = H; a.I = I;

  const int tgu = tile_bytes(bits, H), tdn = tile_bytes(bits, I);
  a.slot_bytes = ((tgu > tdn ? tgu : tdn) + 127) & ~127;
  int limb_x = T * H * 3, limb_h = FD_MAXT * I * 3;
  a.limb_bytes = ((limb_x > limb_h ? limb_x : limb_h) + 127) & ~127;
  int lsc_x = T * (H / 32), lsc_h = (a.limb_bytes / (I * 3)) * (I / 32);
  a.lsc_count = lsc_x > lsc_h ? lsc_x : lsc_h;
  // Ring depth S and consumer warps NA (S a multiple of NA): as many consumer
  // warps as possible, then the deepest ring that fits.
  const size_t cap = max_smem_optin();
  int S = 0, NA = 0;
  for (int s2 = 16; s2 >= 2; --s2) {
    if (smem_layout(s2, a.slot_bytes, a.limb_bytes, a.lsc_count).total > cap) continue;
    int na = NCW;
    while (s2 % na) --na;
    if (na > NA) {
      NA = na;
      S = s2;
    }
  }
  if (S < 2) return QMOE_ERR_UNSUPPORTED;
  a.nslots = S;
  a.ncons = NA;
  size_t smem = smem_layout(S, a.slot_bytes, a.limb_bytes, a.lsc_count).total;

  const void *fn = (bits == 2) ? (const void *)ffn_decode_kernel<2> : (const void *)ffn_decode_kernel<4>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return QMOE_ERR_CUDA;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)num_sms());
  cfg.blockDim = dim3(FD_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // One CTA per SM (shared memory caps residency at one) and a grid of exactly
  // the SM count, so every CTA is resident for the grid barriers; the
  // programmatic-serialization attribute lets this grid launch while the
  // previous kernel drains (the kernel waits for it before reading inputs).
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cooperative) {
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (bits == 2)
    e = cudaLaunchKernelEx(&cfg, ffn_decode_kernel<2>, a);
  else
    e = cudaLaunchKernelEx(&cfg, ffn_decode_kernel<4>, a);
  note_launch();
  return cuda_status(e);
}

extern "C" qmoe_status qmoe_ffn_decode(const qmoe_experts *ex, const float *x, int T, const int32_t *idx,
                                       const float *gate, int k, float *y, void *workspace, size_t workspace_bytes,
                                       int32_t *dev_status, qmoe_stream_t stream) {
  return qmoe::ffn_decode_launch(ex, x, T, idx, gate, k, y, workspace, workspace_bytes, dev_status,
                                 (cudaStream_t)stream, false);
}
