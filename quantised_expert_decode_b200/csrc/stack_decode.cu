// Fused single-token decode stack: all L layers of router -> expert FFN ->
// gate-weighted combine -> residual RMSNorm in ONE persistent kernel (one CTA
// per SM, every CTA resident), so the instruction stream, the shared-memory
// carve-up and the bulk-copy ring stay warm across layers and a layer costs two
// grid barriers instead of several kernel boundaries.
//
// Work split per layer l (G CTAs; CTA c < H/16 owns output rows R_c = 16c..16c+15):
//   A  every CTA: x_l = z_l / rms_l from the z slices and the exact sum of
//      squares of the previous layer; router logits from the exact partial sums
//      of the previous layer (divided by rms_l, plus the bias); top-k with
//      renormalised gates (one warp, identical in every CTA); then the producer
//      warp issues this layer's weight copies.
//   C  gate/up tiles (selected expert j, 16-row tile r, gate or up), one ring
//      item each: a_g = Wg x or a_u = Wu x for those 16 rows -> shared
//      memory. A CTA holds whole 32-row blocks of h (the four tiles gate and
//      up of rows 32b..32b+31), so the warp that completes a block's fourth
//      tile forms h = silu(a_g) * a_u from shared memory, quantises it into
//      limbs and writes them to global (one block quantised once, by one warp)
//      ---- grid barrier (h limbs complete) ----
//   D  row owners: the limbs of every h_j in one bulk copy, down tiles of rows R_c for every selected
//      expert (prefetched during C), y[R_c] = sum_j g_j * (Wd_j h_j)[R_c] in
//      slot order, z_{l+1}[R_c] = x_l[R_c] + y[R_c]; then, from the rows
//      R_c of the next layer's transposed router (prefetched), partial logits
//      sum_{h in R_c} Wr_{l+1}[e][h] z[h] for every expert and the partial sum of
//      squares of z; R_c is one 16-element slice, so both are the slice
//      partials of decode_canon.cuh, added as pairs of integers so the totals
//      are exact and independent of the order of the additions.
//      ---- grid barrier (z, logit and norm partials complete) ----
// The router logit of the next layer is Wr (z / rms) = (Wr z) / rms, which is
// why the partial logits can be formed before the norm is known. Layer 0 uses
// the raw input (no norm); after the last layer x_out = z_L / rms_L.
#include <vector>

#include "common.cuh"
#include "decode_canon.cuh"
#include "decode_tile.cuh"
#include "layout.cuh"
#include "route_common.cuh"
#include "stack_fused.cuh"

namespace qmoe {
namespace {
using namespace tile;

// Consumer warps. With the producer, 12 warps: three per SM sub-partition, so
// up to 168 registers a thread. The legacy integer MMA issues at a fraction of
// the tcgen05 rate and one warp keeps only a couple in flight, so the tile
// dot products want warps more than registers: with 11 consumers a CTA's 8
// gate/up tiles and 10 down tiles each get a warp of their own.
constexpr int SK_NCW = 11;
constexpr int SK_THREADS = 32 * (SK_NCW + 1);
constexpr int SK_MAXK = 16;
constexpr int TRACE_POINTS = 12;
// Trace points of a layer (SM clock of the CTA's consumer thread 0): layer
// start; top-k done; gate/up tiles start; gate/up tiles done (all consumer
// warps); first grid barrier passed; down tiles and partials done; second
// grid barrier passed; logits and normalised x ready (before the top-k);
// first gate/up tile landed (consumer warp 0); h limbs landed; down tiles
// done; z and its sum of squares written (before the next layer's partials).
enum {
  TP_START = 0, TP_TOPK, TP_TILES, TP_TILES_DONE, TP_BAR1, TP_DOWN_DONE, TP_BAR2, TP_LOGITS,
  TP_FIRST_TILE, TP_LIMBS, TP_DOWN_TILES, TP_Z
};
// z and its slice sums of squares are written in Z_COPIES copies and CTA c
// reads copy c % Z_COPIES: every CTA reads all of them right after a grid
// barrier, and fewer readers per cache line shorten phase A.
constexpr int Z_COPIES = 4;
constexpr int CONS_BAR = 1;   // the consumer warps
constexpr int PLAN_BAR = 2;   // consumer warp 0 and the producer warp

struct StackArgs {
  int L, E, H, I, k;
  float eps;
  const uint8_t *const *gu;   // [L] packed gate/up tiles per layer
  const uint8_t *const *dn;   // [L] packed down tiles per layer
  const float *const *bias;   // [L], entries may be null
  const int32_t *fmt;         // [L] block format per layer (read when the kernel's BITS is 0)
  const float *wrt;           // [L][H][E] routers, transposed
  const float *x_in;          // [H]
  float *x_out;               // [H]
  int32_t *idx_rec;           // [L][k]
  float *gate_rec;            // [L][k]
  float *zbuf;                // [Z_COPIES][2 parity][H]
  unsigned long long *lacc;   // [2 parity][E] integer partial-logit sums (2^-32 units, two's complement)
  double *ssq;                // [Z_COPIES][2 parity][H/16] slice sums of squares
  uint8_t *lbuf;              // [k][I/32][LIMB_REC]: limbs of h
  float2 *lscg;               // [k][I/32]: (s, s * sum X) of h's blocks
  unsigned *bar;
  int32_t *status;
  long long *trace;           // [L][G][TRACE_POINTS] SM clock stamps (consumer thread 0), or null
  int nslots, slot_bytes;
  int ncons;                  // consumer warps that take ring items; nslots is a multiple of it
  int w_rows, w_free;         // gate/up work weights of CTAs with / without output rows
};

struct SkState {
  int abort;
  int acq;   // gate/up ring items acquired by the consumer warps so far (all layers)
  int idx[SK_MAXK];
  float gate[SK_MAXK];
  float ztmp[16];
  int vid[SK_MAXK];  // vector ids 0..k-1 of the limb region
  TopkScratch tks;
};

struct SkLayout {
  size_t ring, dnbuf, wrtbuf, xs, limbs, lsc, logits, keys, ytmp, hloc, bars, state, total;
};

// Blocks of h a CTA of a G-CTA grid holds at most (each: a_g and a_u of 32 rows,
// then a completion counter).
__host__ __device__ inline int sk_max_local_blocks(int k, int I, int G) { return (k * (I / 32) + G - 1) / G; }
constexpr int HLOC_BYTES = 2 * 32 * 4 + 16;

__host__ __device__ inline size_t al128(size_t v) { return (v + 127) & ~(size_t)127; }

__host__ __device__ inline SkLayout sk_layout(int bits, int E, int H, int I, int k, int nslots, int slot_bytes,
                                               int G) {
  SkLayout o;
  const size_t tdn = (size_t)tile_bytes(bits, I);
  const size_t vecs = (size_t)((H / 32) > k * (I / 32) ? (H / 32) : k * (I / 32));  // limb records
  o.ring = 0;
  o.dnbuf = al128(o.ring + (size_t)nslots * slot_bytes);
  o.wrtbuf = al128(o.dnbuf + (size_t)k * tdn);
  const size_t wrt_bytes = (size_t)16 * E * 4, key_bytes = (size_t)32 * topk_m(E) * 4;
  o.xs = al128(o.wrtbuf + (wrt_bytes > key_bytes ? wrt_bytes : key_bytes));
  o.limbs = al128(o.xs + (size_t)H * 4);
  o.lsc = al128(o.limbs + vecs * LIMB_REC);
  o.logits = al128(o.lsc + vecs * 8);
  // The key table of the top-k is live only in phase A, while the router-row
  // buffer is idle (its last reads were in the previous layer's phase D, its
  // next fill is issued after the layer's gate/up tiles): they share memory.
  o.keys = o.wrtbuf;
  o.ytmp = al128(o.logits + (size_t)E * 8);
  o.hloc = al128(o.ytmp + (size_t)k * 16 * 4);
  o.bars = al128(o.hloc + (size_t)sk_max_local_blocks(k, I, G) * HLOC_BYTES);
  o.state = al128(o.bars + (size_t)(2 * nslots + 3) * 8);
  o.total = o.state + sizeof(SkState);
  return o;
}

// Adds one slice partial to an exact integer total; false when the partial is
// out of the fixed-point range.
__device__ __forceinline__ bool add_fixed(unsigned long long *acc, double p) {
  long long v;
  const bool ok = canon::fix(p, v);
  atomicAdd(acc, (unsigned long long)v);
  return ok;
}

// Consumer-side grid barrier: the 256 consumer threads meet, one thread joins
// the grid, the consumers meet again. Returns false once the CTA has aborted.
__device__ __forceinline__ void trace_point(const StackArgs &a, int l, int p) {
  if (a.trace) a.trace[((size_t)l * gridDim.x + blockIdx.x) * TRACE_POINTS + p] = clock64();
}

__device__ __forceinline__ bool cons_grid_barrier(const StackArgs &a, SkState *st, int tid, int l = -1,
                                                  int p_before = 0) {
  named_barrier_sync(CONS_BAR, SK_NCW * 32);
  if (tid == 0) {
    if (l >= 0) trace_point(a, l, p_before);
    if (!*(volatile int *)&st->abort && !grid_barrier_one_thread(a.bar, gridDim.x)) {
      set_status(a.status, DEV_TIMEOUT);
      *(volatile int *)&st->abort = 1;
    }
    __threadfence();
    if (l >= 0) trace_point(a, l, p_before + 1);
  }
  named_barrier_sync(CONS_BAR, SK_NCW * 32);
  return !*(volatile int *)&st->abort;
}

// Top-k of logits held in shared memory (kept out of line: it runs once per
// layer and would otherwise add its registers to the kernel body's).
__device__ __noinline__ void topk_smem(const double *logits, const unsigned *keys, int E, int k, int32_t *idx,
                                       float *gate, TopkScratch *sc) {
  switch (topk_m(E)) {
    case 4: warp_topk_table_m<4>(logits, keys, E, k, idx, gate, sc); break;
    case 8: warp_topk_table_m<8>(logits, keys, E, k, idx, gate, sc); break;
    case 16: warp_topk_table_m<16>(logits, keys, E, k, idx, gate, sc); break;
    default: warp_topk_table_m<32>(logits, keys, E, k, idx, gate, sc); break;
  }
}

// One warp: h = silu(a_g) * a_u for the 32 rows of block b of selected
// expert j (lane i: row 32b + i) from the block's a_g / a_u in shared memory,
// quantised exactly as every decode path quantises a 32-element block; limbs
// and scales go to global for the row owners.
__device__ __noinline__ void quant_h_block(const StackArgs &a, const float *hl, int j, int b, int lane) {
  const int nblkI = a.I / 32;
  const float h = canon::hval(hl[lane], hl[32 + lane]);
  float m = fabsf(h);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sc, inv;
  block_scale(m, sc, inv);
  const int X = quant_one(h, inv);
  int l[3];
  limbs3(X, l[0], l[1], l[2]);
  uint8_t *rec = a.lbuf + ((size_t)j * nblkI + b) * LIMB_REC;
#pragma unroll
  for (int p = 0; p < 3; ++p) {   // lanes 4q..4q+3 -> one little-endian word
    const uint32_t v = (uint32_t)(l[p] & 0xff);
    const uint32_t w = v | (__shfl_down_sync(0xffffffffu, v, 1) << 8) | (__shfl_down_sync(0xffffffffu, v, 2) << 16) |
                       (__shfl_down_sync(0xffffffffu, v, 3) << 24);
    if ((lane & 3) == 0) *reinterpret_cast<uint32_t *>(rec + p * 32 + lane) = w;
  }
  int sx = X;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
  if (lane == 0) a.lscg[(size_t)j * nblkI + b] = make_float2(sc, __fmul_rn(sc, (float)sx));
}

// A tile's dot product in the layer's block format: BITS when the stack has
// one format, else the layer's own (bl).
template <int BITS>
__device__ __forceinline__ float2 tile_dot_fmt(int bl, const uint8_t *tile, int nblk, const uint8_t *limbs,
                                               const float2 *lsc) {
  if constexpr (BITS != 0) {
    return tile_dot1<BITS, 1>(tile, nblk, limbs, lsc);
  } else {
    return bl == QMOE_Q2 ? tile_dot1<QMOE_Q2, 1>(tile, nblk, limbs, lsc) : tile_dot1<QMOE_Q4, 1>(tile, nblk, limbs, lsc);
  }
}

// BITS: the stack's block format, or 0 for a stack whose layers mix formats
// (shared memory laid out for the widest, Q4; tile sizes per layer).
template <int BITS>
__global__ void __launch_bounds__(SK_THREADS, 1) stack_decode_kernel(StackArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = a.nslots;
  const int H = a.H, I = a.I, E = a.E, k = a.k, L = a.L;
  const SkLayout lay = sk_layout(BITS ? BITS : QMOE_Q4, E, H, I, k, S, a.slot_bytes, (int)gridDim.x);
  uint8_t *ring = smem + lay.ring;
  uint8_t *dnbuf = smem + lay.dnbuf;
  float *wrtbuf = reinterpret_cast<float *>(smem + lay.wrtbuf);
  float *xs = reinterpret_cast<float *>(smem + lay.xs);
  uint8_t *limbs = smem + lay.limbs;
  float2 *lsc = reinterpret_cast<float2 *>(smem + lay.lsc);
  double *logits = reinterpret_cast<double *>(smem + lay.logits);
  unsigned *keytab = reinterpret_cast<unsigned *>(smem + lay.keys);
  const int MK = topk_m(E);
  float *ytmp = reinterpret_cast<float *>(smem + lay.ytmp);
  uint8_t *hloc = smem + lay.hloc;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.bars);
  uint64_t *empty = full + S;
  uint64_t *dnbar = empty + S;
  uint64_t *wrtbar = dnbar + 1;
  uint64_t *hbar = wrtbar + 1;
  SkState *st = reinterpret_cast<SkState *>(smem + lay.state);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nblkH = H / 32, nblkI = I / 32, I16 = I / 16, H16 = H / 16;
  const int tgu0 = tile_bytes(BITS ? BITS : QMOE_Q4, H), tdn0 = tile_bytes(BITS ? BITS : QMOE_Q4, I);
  const int G = (int)gridDim.x, c = blockIdx.x;
  const bool rows = c < H16;
  const int r0 = 16 * c;
  // gate/up items (selected expert j, matrix gate or up, 16-row tile r) of this
  // CTA: item i = 2 (j I16 + r) + matrix, so the four items 4B..4B+3 are the
  // gate and up tiles of the 32-row block B = j (I/32) + b of h. A CTA takes
  // whole blocks (1 or 2 of the 240 at the 512-expert shape), so each block
  // of h is formed and quantised where its tiles were computed.
  auto wcum = [&](int cc) -> long long {
    const int nr = cc < H16 ? cc : H16;
    return (long long)nr * a.w_rows + (long long)(cc - nr) * a.w_free;
  };
  const int NBLK = k * nblkI;
  const long long WT = wcum(G);
  const int blo = (int)(wcum(c) * NBLK / WT), bhi = (int)(wcum(c + 1) * NBLK / WT);
  const int ilo = 4 * blo, ihi = 4 * bhi;
  const int nitems = ihi - ilo;
  const int nth = SK_NCW * 32;
  const bool producer = warp == SK_NCW;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(dnbar, 1);
    mbar_init(wrtbar, 1);
    mbar_init(hbar, 1);
    fence_mbar_init();
    st->abort = 0;
    st->acq = 0;
    for (int q = 0; q < sk_max_local_blocks(k, I, G); ++q)
      *reinterpret_cast<int *>(hloc + q * HLOC_BYTES + 256) = 0;
    for (int j = 0; j < SK_MAXK; ++j) st->vid[j] = j;
  }
  __syncthreads();

  // ------------------------------------------ prologue: layer-0 logit partials
  if (producer && lane == 0 && rows) {
    mbar_arrive_expect_tx(wrtbar, (uint32_t)(16 * E * 4));
    bulk_g2s(wrtbuf, a.wrt + (size_t)r0 * E, (uint32_t)(16 * E * 4), wrtbar);
  }
  if (!producer && rows) {
    if (tid < 16) {
      const float z = a.x_in[r0 + tid];
      st->ztmp[tid] = z;
      for (int cp = 0; cp < Z_COPIES; ++cp) a.zbuf[(size_t)cp * 2 * H + r0 + tid] = z;
    }
    named_barrier_sync(CONS_BAR, nth);
    if (!mbar_wait(wrtbar, 0u, clock64() + WAIT_BUDGET_CYCLES)) {
      set_status(a.status, DEV_TIMEOUT);
      st->abort = 1;
    } else {
      bool ok = true;
      double zd[canon::SLICE];
#pragma unroll
      for (int i = 0; i < canon::SLICE; ++i) zd[i] = canon::f2d(st->ztmp[i]);
      for (int e = tid; e < E; e += nth)
        ok &= add_fixed(&a.lacc[e], canon::slice_dot_wide([&](int i) { return wrtbuf[i * E + e]; }, zd));
      if (!ok) set_status(a.status, DEV_RANGE);
    }
  }
  if (!producer) cons_grid_barrier(a, st, tid);

  // Ring bookkeeping shared by producer and consumers (same sequence of items).
  // Item n goes to slot n % S; within a layer the m-th item of the CTA goes
  // to consumer warp m % NA, and S is a multiple of NA, so a slot's phases of
  // one layer are taken in order by one warp (and its phase of the previous
  // layer completed before the layer's grid barriers): when a warp waits for
  // item n the slot's barrier is in the phase of item n, and the parity wait
  // is exact.
  int nring = 0;
  const int NA = a.ncons;
  auto wait_full = [&](int n) -> bool {
    const long long dl = clock64() + WAIT_BUDGET_CYCLES;
    const uint32_t par = (uint32_t)((n / S) & 1);
    while (!mbar_try_wait(&full[n % S], par)) {
      if (*(volatile int *)&st->abort) return false;
      if (clock64() > dl) {
        set_status(a.status, DEV_TIMEOUT);
        *(volatile int *)&st->abort = 1;
        return false;
      }
    }
    __syncwarp();
    if (lane == 0) atomicAdd(&st->acq, 1);
    return true;
  };

  for (int l = 0; l < L; ++l) {
    const int par = l & 1;
    const int bl = BITS ? BITS : __ldg(a.fmt + l);
    const int tgu = BITS ? tgu0 : tile_bytes(bl, H), tdn = BITS ? tdn0 : tile_bytes(bl, I);
    if (tid == 0) {
      trace_point(a, l, TP_START);
      // points of phases a CTA has no work in stay 0
      if (a.trace && nitems == 0) a.trace[((size_t)l * gridDim.x + blockIdx.x) * TRACE_POINTS + TP_FIRST_TILE] = 0;
      if (a.trace && !rows)
        for (int q = TP_LIMBS; q <= TP_Z; ++q) a.trace[((size_t)l * gridDim.x + blockIdx.x) * TRACE_POINTS + q] = 0;
    }
    // ------------------------------------------------------------------ A --
    if (!producer && !*(volatile int *)&st->abort) {
      // one batch of loads: sum of squares, z, partial logits, bias
      const int zc = c % Z_COPIES;
      const float4 *zb = reinterpret_cast<const float4 *>(a.zbuf + ((size_t)zc * 2 + par) * H);
      const float *b = a.bias[l];
      const unsigned long long *la = a.lacc + (size_t)par * E;
      float4 zv[4];
      unsigned long long lh[4];
      float bv[4];
      const double *sq = a.ssq + ((size_t)zc * 2 + par) * H16;
      double sv[4];   // this lane's first slice sums of squares (decode_canon.cuh's order)
#pragma unroll
      for (int m = 0; m < 4; ++m) sv[m] = (l > 0 && lane + 32 * m < H16) ? __ldcg(sq + lane + 32 * m) : 0.0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = tid + i * nth;
        if (q < H / 4) zv[i] = __ldcg(zb + q);
        if (q < E) {
          lh[i] = __ldcg(la + q);
          bv[i] = b ? __ldg(b + q) : 0.0f;
        }
      }
      // every warp adds the slice sums of squares itself (same order, same value)
      const double rinv =
          l > 0 ? canon::norm_rinv(canon::warp_sum_slices<4>(sv, [&](int cc) { return __ldcg(sq + cc); }, H16), H,
                                   a.eps)
                : 1.0;
      const float inv = __double2float_rn(rinv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = tid + i * nth;
        if (q < H / 4) {
          float4 v = zv[i];
          if (l > 0) {
            v.x = __fmul_rn(v.x, inv); v.y = __fmul_rn(v.y, inv); v.z = __fmul_rn(v.z, inv); v.w = __fmul_rn(v.w, inv);
          }
          reinterpret_cast<float4 *>(xs)[q] = v;
        }
        if (q < E) {
          const double lv = canon::logit(canon::unfix((long long)lh[i]), rinv, canon::f2d(bv[i]));
          logits[q] = lv;
          keytab[key_slot(q, MK)] = logit_key(lv);
        }
      }
      for (int q = tid + 4 * nth; q < H / 4; q += nth) {   // larger geometries only
        float4 v = __ldcg(zb + q);
        if (l > 0) {
          v.x = __fmul_rn(v.x, inv); v.y = __fmul_rn(v.y, inv); v.z = __fmul_rn(v.z, inv); v.w = __fmul_rn(v.w, inv);
        }
        reinterpret_cast<float4 *>(xs)[q] = v;
      }
      for (int q = tid + 4 * nth; q < E; q += nth) {
        const double lv = canon::logit(canon::unfix((long long)__ldcg(la + q)), rinv, b ? canon::f2d(b[q]) : 0.0);
        logits[q] = lv;
        keytab[key_slot(q, MK)] = logit_key(lv);
      }
      // clear the other parity's accumulators for the next layer (read last by
      // every CTA before the previous barriers)
      unsigned long long *lz = a.lacc + (size_t)(par ^ 1) * E;
      for (int e = c * nth + tid; e < E; e += G * nth) lz[e] = 0ull;
      named_barrier_sync(CONS_BAR, nth);
      if (tid == 0) trace_point(a, l, TP_LOGITS);
      if (warp == 0) {
        topk_smem(logits, keytab, E, k, st->idx, st->gate, &st->tks);
        if (lane == 0) trace_point(a, l, TP_TOPK);
        // the selection always names k distinct experts in [0, E) (NaN logits
        // rank lowest); checked anyway before any address is formed from it
        if (lane < k && (unsigned)st->idx[lane] >= (unsigned)E) {
          set_status(a.status, DEV_BAD_INDEX);
          *(volatile int *)&st->abort = 1;
        }
        __syncwarp();
        if (c == 0 && lane < k) {
          a.idx_rec[l * k + lane] = st->idx[lane];
          a.gate_rec[l * k + lane] = st->gate[lane];
        }
      } else {
        // quantise x_l (all 7 other warps)
        const int nch = H / 128;
        for (int task = warp - 1; task < nch; task += SK_NCW - 1) {
          const float4 v = reinterpret_cast<const float4 *>(xs + task * 128)[lane];
          quant_chunk_inl(v, limbs, lsc, task, lane);
        }
      }
    }
    // Warp 0 hands the selection to the producer as soon as its top-k is done,
    // while the other consumer warps still quantise x. Both sides read one
    // abort value: nothing sets it between here and the consumer barrier below.
    if (warp == 0 || producer) named_barrier_sync(PLAN_BAR, 64);
    if (producer && *(volatile int *)&st->abort) break;

    if (producer) {
      // -------------------------------------------------------------- B --
      // lane s < S: ring slot s (gate/up tiles, in item order); lane 31: this
      // CTA's down tiles; lane 30: next layer's router rows.
      fence_proxy_async();   // ring memory was last read with ordinary loads
      const uint8_t *gu = a.gu[l];
      const uint64_t pol = l2_evict_first();
      const int first = nring + ((lane - nring % S) % S + S) % S;  // first item of slot `lane`
      for (int n = first; lane < S && n < nring + nitems; n += S) {
        const int s = n % S;
        if (n >= S) {
          const long long dl = clock64() + WAIT_BUDGET_CYCLES;
          bool ok = true;
          while (!mbar_try_wait(&empty[s], (uint32_t)(((n / S) - 1) & 1))) {
            if (*(volatile int *)&st->abort || clock64() > dl) {
              ok = false;
              break;
            }
          }
          if (!ok) break;
        }
        const int i = ilo + (n - nring), u = i >> 1, mat = i & 1;
        const int j = u / I16, r = u % I16;
        const uint8_t *src = gu + (((size_t)st->idx[j] * 2 + mat) * I16 + r) * (size_t)tgu;
        mbar_arrive_expect_tx(&full[s], (uint32_t)tgu);
        bulk_g2s_hint(ring + (size_t)s * a.slot_bytes, src, (uint32_t)tgu, &full[s], pol);
      }
      if ((lane == 31 || lane == 30) && rows) {
        // The down tiles and the next layer's router rows are needed only after
        // the h barrier: issue them once this CTA's gate/up tiles have landed
        // (every ring item of the layer acquired), so that they do not compete
        // with the gate/up stream on the critical path.
        const int want = nring + nitems;
        const long long dl = clock64() + WAIT_BUDGET_CYCLES;
        bool ok = true;
        while (*(volatile int *)&st->acq < want) {
          if (*(volatile int *)&st->abort) {
            ok = false;
            break;
          }
          if (clock64() > dl) {
            set_status(a.status, DEV_TIMEOUT);
            *(volatile int *)&st->abort = 1;
            ok = false;
            break;
          }
          __nanosleep(64);
        }
        if (ok && lane == 31) {
          const uint8_t *dn = a.dn[l];
          mbar_arrive_expect_tx(dnbar, (uint32_t)(k * tdn));
          for (int j = 0; j < k; ++j)
            bulk_g2s_hint(dnbuf + (size_t)j * tdn, dn + ((size_t)st->idx[j] * H16 + c) * (size_t)tdn, (uint32_t)tdn,
                          dnbar, pol);
        }
        if (ok && lane == 30 && l + 1 < L) {
          mbar_arrive_expect_tx(wrtbar, (uint32_t)(16 * E * 4));
          bulk_g2s_hint(wrtbuf, a.wrt + ((size_t)(l + 1) * H + r0) * E, (uint32_t)(16 * E * 4), wrtbar, pol);
        }
      }
      nring += nitems;
      continue;
    }

    named_barrier_sync(CONS_BAR, nth);   // x limbs complete
    if (*(volatile int *)&st->abort) break;
    if (tid == 0) trace_point(a, l, TP_TILES);

    // -------------------------------------------------------------------- C --
    // Each consumer warp first asks L2 for its own items with ordinary
    // prefetches. They travel the load path beside the producer's bulk copies
    // of the same bytes, so more of the layer's weights are in flight per SM.
    for (int m = warp; warp < NA && m < nitems; m += NA) {
      const int i = ilo + m, u = i >> 1, mat = i & 1, j = u / I16, r = u % I16;
      const uint8_t *src = a.gu[l] + (((size_t)st->idx[j] * 2 + mat) * I16 + r) * (size_t)tgu;
      for (int off = lane * 128; off < tgu; off += 32 * 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(src + off));
    }
    for (int m = warp; warp < NA && m < nitems; m += NA) {
      const int n = nring + m;
      if (!wait_full(n)) break;
      if (tid == 0 && m == 0) trace_point(a, l, TP_FIRST_TILE);
      const int i = ilo + m, u = i >> 1, mat = i & 1, j = u / I16, r = u % I16;
      const float2 o = tile_dot_fmt<BITS>(bl, ring + (size_t)(n % S) * a.slot_bytes, nblkH, limbs, lsc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[n % S]);
      // this tile's 16 rows into the local block: a_g / a_u of rows 16 (r & 1) ..
      float *hl = reinterpret_cast<float *>(hloc + ((i >> 2) - blo) * HLOC_BYTES);
      if ((lane & 3) == 0) {   // lanes of quad g hold rows g and g+8 of the tile
        const int g = lane >> 2;
        hl[mat * 32 + (r & 1) * 16 + g] = o.x;
        hl[mat * 32 + (r & 1) * 16 + g + 8] = o.y;
      }
      // the warp that completes the block's fourth tile quantises the block
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = atomicAdd(reinterpret_cast<int *>(hl + 64), 1) == 3;
        if (last) {
          __threadfence_block();
          *reinterpret_cast<volatile int *>(hl + 64) = 0;   // for the next layer
        }
      }
      if (__shfl_sync(0xffffffffu, last, 0)) {
        __syncwarp();
        quant_h_block(a, hl, j, r >> 1, lane);
      }
    }
    nring += nitems;
    if (!cons_grid_barrier(a, st, tid, l, TP_TILES_DONE)) continue;

    // -------------------------------------------------------------------- D --
    if (rows) {
      {
        // the limbs and block scales of every selected expert's h (quantised
        // during C) arrive in two bulk copies
        const uint32_t lbytes = (uint32_t)(k * nblkI * LIMB_REC), sbytes = (uint32_t)(k * nblkI * 8);
        if (tid == 0) {
          fence_proxy_async();   // global limbs were written by ordinary stores; smem limbs read by ordinary loads
          mbar_arrive_expect_tx(hbar, lbytes + sbytes);
          bulk_g2s(limbs, a.lbuf, lbytes, hbar);
          bulk_g2s(lsc, a.lscg, sbytes, hbar);
        }
        if (!mbar_wait(hbar, (uint32_t)(l & 1), clock64() + WAIT_BUDGET_CYCLES)) {
          set_status(a.status, DEV_TIMEOUT);
          *(volatile int *)&st->abort = 1;
        }
        if (tid == 0) trace_point(a, l, TP_LIMBS);
      }
      named_barrier_sync(CONS_BAR, nth);
      bool ok = mbar_wait(dnbar, (uint32_t)(l & 1), clock64() + WAIT_BUDGET_CYCLES);
      if (ok) {
        for (int j = warp; j < k; j += SK_NCW) {
          const float2 o = tile_dot_fmt<BITS>(bl, dnbuf + (size_t)j * tdn, nblkI,
                                              limbs + (size_t)j * nblkI * LIMB_REC, lsc + (size_t)j * nblkI);
          if ((lane & 3) == 0) {
            const int g = lane >> 2;
            ytmp[j * 16 + g] = o.x;
            ytmp[j * 16 + g + 8] = o.y;
          }
        }
      } else {
        set_status(a.status, DEV_TIMEOUT);
        *(volatile int *)&st->abort = 1;
      }
      named_barrier_sync(CONS_BAR, nth);
      if (tid == 0) trace_point(a, l, TP_DOWN_TILES);
      if (ok && warp == 0) {
        if (lane < 16) {
          float y = 0.0f;
          for (int j = 0; j < k; ++j) y = canon::combine_step(y, st->gate[j], ytmp[j * 16 + lane]);  // slot order
          const float z = __fadd_rn(xs[r0 + lane], y);
          st->ztmp[lane] = z;
#pragma unroll
          for (int cp = 0; cp < Z_COPIES; ++cp) a.zbuf[((size_t)cp * 2 + (par ^ 1)) * H + r0 + lane] = z;
        }
        __syncwarp();
        if (lane < Z_COPIES)
          a.ssq[((size_t)lane * 2 + (par ^ 1)) * H16 + c] = canon::slice_sumsq([&](int i) { return st->ztmp[i]; });
      }
      named_barrier_sync(CONS_BAR, nth);
      if (tid == 0) trace_point(a, l, TP_Z);
      if (ok && l + 1 < L) {
        if (mbar_wait(wrtbar, (uint32_t)((l + 1) & 1), clock64() + WAIT_BUDGET_CYCLES)) {
          unsigned long long *la = a.lacc + (size_t)(par ^ 1) * E;
          bool rok = true;
          double zd[canon::SLICE];
#pragma unroll
          for (int i = 0; i < canon::SLICE; ++i) zd[i] = canon::f2d(st->ztmp[i]);
          for (int e = tid; e < E; e += nth)
            rok &= add_fixed(la + e, canon::slice_dot_wide([&](int i) { return wrtbuf[i * E + e]; }, zd));
          if (!rok) set_status(a.status, DEV_RANGE);
        } else {
          set_status(a.status, DEV_TIMEOUT);
          *(volatile int *)&st->abort = 1;
        }
      }
    }
    cons_grid_barrier(a, st, tid, l, TP_DOWN_DONE);
  }

  if (producer) {
    // never leave with copies in flight (only after an abort can any remain)
    if (lane < S && *(volatile int *)&st->abort) {
      const long long dl = clock64() + WAIT_BUDGET_CYCLES;
      for (int n = nring + lane - S; n < nring; n += S)
        if (n >= 0)
          while (!mbar_try_wait(&full[n % S], (uint32_t)((n / S) & 1)))
            if (clock64() > dl) break;
    }
    return;
  }
  if (*(volatile int *)&st->abort) return;
  // ---------------------------------------------------------------- output --
  if (rows && warp == 0) {
    const double *sq = a.ssq + (size_t)(L & 1) * H16;
    const double ss = canon::warp_sumsq([&](int cc) { return __ldcg(sq + cc); }, H16);
    const float inv = __double2float_rn(canon::norm_rinv(ss, H, a.eps));
    if (lane < 16) a.x_out[r0 + lane] = __fmul_rn(__ldcg(a.zbuf + (size_t)(L & 1) * H + r0 + lane), inv);
  }
  // leave lacc[0] clear for the next launch's layer-0 partials (its last
  // reader finished long before the last barrier)
  for (int e = c * nth + tid; e < E; e += G * nth) a.lacc[e] = 0ull;
}

}  // namespace

// ---------------------------------------------------------------- host side --
// Can the fused kernel run this stack? Fills the launch plan when it can.
bool fused_stack_plan(int fmt, int E, int H, int I, int k, FusedPlan *p) {
  if (k > SK_MAXK || E > 1024 || H / 16 > num_sms() || H % 128 || I % 128) return false;
  // As many consumer warps taking ring items as possible (the ring depth a
  // multiple of their number), then the deepest ring that fits.
  const int slot = (int)al128((size_t)tile_bytes(fmt, H));
  const size_t cap = max_smem_optin();
  int best_na = 0;
  for (int S = 14; S >= 4; --S) {
    const SkLayout o = sk_layout(fmt, E, H, I, k, S, slot, num_sms());
    if (o.total > cap) continue;
    int na = SK_NCW;
    while (S % na) --na;
    if (na > best_na) {
      best_na = na;
      p->smem = o.total;
      p->nslots = S;
      p->ncons = na;
      p->slot_bytes = slot;
    }
  }
  return best_na > 0;
}

size_t fused_stack_ws_bytes(int L, int E, int H, int I, int k) {
  auto a = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const size_t nb = (size_t)k * (I / 32);
  return a((size_t)L * H * E * 4) + a(2 * (size_t)E * 8) + a(Z_COPIES * 2 * (size_t)(H / 16) * 8) + a(Z_COPIES * 2 * (size_t)H * 4) +
         a(nb * LIMB_REC) + a(nb * 8) + 256 + 3 * a((size_t)L * 8) + a((size_t)L * 4);
}


FusedBufs fused_carve(void *ws, int L, int E, int H, int I, int k) {
  auto a = [](size_t v) { return (v + 255) & ~(size_t)255; };
  char *p = static_cast<char *>(ws);
  FusedBufs b;
  b.wrt = reinterpret_cast<float *>(p); p += a((size_t)L * H * E * 4);
  b.lacc = reinterpret_cast<unsigned long long *>(p); p += a(2 * (size_t)E * 8);
  b.ssq = reinterpret_cast<double *>(p); p += a(Z_COPIES * 2 * (size_t)(H / 16) * 8);
  b.zbuf = reinterpret_cast<float *>(p); p += a(Z_COPIES * 2 * (size_t)H * 4);
  const size_t nb = (size_t)k * (I / 32);
  b.lbuf = reinterpret_cast<uint8_t *>(p); p += a(nb * LIMB_REC);
  b.lscg = reinterpret_cast<float2 *>(p); p += a(nb * 8);
  b.bar = reinterpret_cast<unsigned *>(p); p += 256;
  b.gu = reinterpret_cast<const uint8_t **>(p); p += a((size_t)L * 8);
  b.dn = reinterpret_cast<const uint8_t **>(p); p += a((size_t)L * 8);
  b.bias = reinterpret_cast<const float **>(p); p += a((size_t)L * 8);
  b.fmt = reinterpret_cast<int32_t *>(p);
  return b;
}

namespace {
__global__ void transpose_router(const float *Wr, float *WrT, int E, int H) {
  __shared__ float t[32][33];
  const int e0 = blockIdx.y * 32, h0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y)
    if (e0 + i < E) t[i][threadIdx.x] = Wr[(size_t)(e0 + i) * H + h0 + threadIdx.x];
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y)
    if (e0 + threadIdx.x < E) WrT[(size_t)(h0 + i) * E + e0 + threadIdx.x] = t[threadIdx.x][i];
}
}  // namespace

// Prepare the fused buffers (transposed routers, pointer tables); called once
// at stack creation on `s`.
qmoe_status fused_prepare(const FusedBufs &b, int L, int E, int H, const float *const *Wr,
                          const qmoe_experts *layers, const float *const *bias, cudaStream_t s) {
  for (int l = 0; l < L; ++l) {
    transpose_router<<<dim3(H / 32, (E + 31) / 32), dim3(32, 8), 0, s>>>(Wr[l], b.wrt + (size_t)l * H * E, E, H);
    note_launch();
  }
  std::vector<const void *> gu(L), dn(L), bi(L);
  std::vector<int32_t> fm(L);
  for (int l = 0; l < L; ++l) {
    gu[l] = layers[l].gate_up;
    dn[l] = layers[l].down;
    bi[l] = bias ? bias[l] : nullptr;
    fm[l] = layers[l].fmt;
  }
  if (cudaMemcpyAsync((void *)b.gu, gu.data(), L * 8, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync((void *)b.dn, dn.data(), L * 8, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync((void *)b.bias, bi.data(), L * 8, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync((void *)b.fmt, fm.data(), L * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return QMOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return QMOE_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}

qmoe_status fused_launch(const FusedBufs &b, const FusedPlan &p, int fmt, int L, int E, int H, int I, int k, float eps,
                         const float *x_in, float *x_out, int32_t *idx_rec, float *gate_rec, int32_t *status,
                         long long *trace, cudaStream_t s, bool cooperative) {
  StackArgs a{};
  a.L = L; a.E = E; a.H = H; a.I = I; a.k = k; a.eps = eps;
  a.gu = b.gu; a.dn = b.dn; a.bias = b.bias; a.fmt = b.fmt; a.wrt = b.wrt;
  a.x_in = x_in; a.x_out = x_out; a.idx_rec = idx_rec; a.gate_rec = gate_rec;
  a.zbuf = b.zbuf; a.lacc = b.lacc; a.ssq = b.ssq; a.bar = b.bar; a.status = status;
  a.lbuf = b.lbuf; a.lscg = b.lscg;
  a.trace = trace;
  a.nslots = p.nslots; a.slot_bytes = p.slot_bytes; a.ncons = p.ncons;
  // Gate/up units are split evenly: the h barrier waits for the slowest CTA's
  // gate/up tiles, while the row owners' down tiles and router rows are only
  // needed after it and stream in behind the gate/up work.
  const int G = num_sms();
  a.w_rows = 1;
  a.w_free = 1;
  const void *fn = fmt == QMOE_Q2   ? (const void *)stack_decode_kernel<QMOE_Q2>
                   : fmt == QMOE_Q4 ? (const void *)stack_decode_kernel<QMOE_Q4>
                                    : (const void *)stack_decode_kernel<0>;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem) != cudaSuccess)
    return QMOE_ERR_CUDA;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)G);
  cfg.blockDim = dim3(SK_THREADS);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 1 : 0;
  cudaError_t e = fmt == QMOE_Q2   ? cudaLaunchKernelEx(&cfg, stack_decode_kernel<QMOE_Q2>, a)
                  : fmt == QMOE_Q4 ? cudaLaunchKernelEx(&cfg, stack_decode_kernel<QMOE_Q4>, a)
                                   : cudaLaunchKernelEx(&cfg, stack_decode_kernel<0>, a);
  note_launch();
  return cuda_status(e);
}

}  // namespace qmoe

namespace qmoe {
int fused_trace_points() { return TRACE_POINTS; }
}  // namespace qmoe
