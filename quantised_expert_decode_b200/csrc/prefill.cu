// Prefill expert FFN for chunks of many tokens ([P3] batched prefill in chunks,
// "Understanding the Architecture"): bucketing of the routed (token, slot)
// pairs by expert, a tile plan, and two grouped GEMMs on the fifth-generation
// tensor cores with the Q4 expert weights dequantised to bf16 in shared memory.
//
//   GEMM 1, per expert e and 128 intermediate features f:
//       G = Wg[f,:] X_e^T,  U = Wu[f,:] X_e^T      (fp32 in tensor memory)
//       h[pair, f] = bf16(silu(G) * U)
//   GEMM 2, per expert e and 256 hidden features o:
//       Y = Wd[o,:] h_e^T;  part[pair, o] = gate[pair] * Y  (fp32, bucket order)
//   combine, per token t: y[t, :] = sum over slots j (in slot order) of
//       part[pair (t, j), :]     - every run adds the same terms in the same
//       order, so y is reproducible bit for bit. (The earlier form, fp32
//       atomic additions straight into y, is kept behind a flag of the timed
//       entry point for comparison; its order, and y's last bits, vary.)
// X_e is the bf16 activation rows of the tokens routed to e, gathered by
// token id; h is kept in bucket order with every expert's rows padded to a
// multiple of 16. The weights form the 128-row MMA operand and the tokens the
// N operand (16..PF_N, a multiple of 16), so an expert with n tokens costs
// ceil(n/16)*16 columns, not a 128-row tile. Tensor memory holds two
// accumulator slots of 256 columns: a tile of at most 128 tokens takes one
// (its two accumulators side by side), so the epilogue of one such tile
// overlaps the main loop of the next; a wider tile takes both.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "layout.cuh"
#include "tc05.cuh"

namespace qmoe {

size_t bucket_ws_bytes(int T, int k, int E);
bool bucket_supported(int T, int k, int E);
qmoe_status bucket_launch(const int32_t *idx, const float *gate, int T, int k, int E, void *ws, int32_t *offsets,
                          int32_t *perm, int32_t *ptok, float *pgate, int32_t *active, int32_t *nactive,
                          bool check_dup, int32_t *status, cudaStream_t s);

namespace {

constexpr int PF_N = 256;                               // max tokens per tile (MMA N)
constexpr int PF_M = 128;                               // rows per A operand (MMA M)
constexpr int PF_KS = 64;                               // reduction elements per pipeline step
constexpr int PF_SA = 3;                                // dequantised weight stages (A0 + A1)
constexpr int PF_SB = 3;                                // activation stages (B)
constexpr int PF_PS = 3;                                // packed-weight stages
constexpr int PF_B_PREFETCH = 8;                        // k-steps of activation rows prefetched into L2 ahead
constexpr int PF_A_BYTES = PF_M * PF_KS * 2;            // 16 KB per A operand
constexpr int PF_ASTAGE = 2 * PF_A_BYTES;               // A0 + A1
constexpr int PF_B_BYTES = PF_N * PF_KS * 2;            // 32 KB
constexpr int PF_B_BOX = 64;                            // activation rows per TMA load
constexpr int PF_PK_CODES = 16 * 512;                   // 16 tile groups x 64 Q4 codes x 16 rows
constexpr int PF_PK_SCALES = 16 * 128;                  // 16 tiles x 2 blocks x 16 rows x (d, m)
constexpr int PF_PK = PF_PK_CODES + PF_PK_SCALES;
constexpr int PF_OFF_B = PF_SA * PF_ASTAGE;
constexpr int PF_OFF_PK = PF_OFF_B + PF_SB * PF_B_BYTES;
constexpr int PF_OFF_BAR = PF_OFF_PK + PF_PS * PF_PK;
constexpr int PF_SMEM = PF_OFF_BAR + 256 + 1024;        // barriers + alignment slack
constexpr int PF_PREFETCH = 16;                         // k-steps of packed weights prefetched into L2 ahead
constexpr int PF_PF_BOX = 8;                            // k-steps per L2 prefetch
constexpr int PF_TMEM_COLS = 512;
constexpr int PF_SLOT = PF_TMEM_COLS / 2;               // columns of one accumulator slot
constexpr int PF_NARROW = PF_SLOT / 2;                  // widest tile that fits one slot
constexpr int PF_MAX_E = 1024;

// warp roles
constexpr int W_PRODUCER = 0;   // TMA loads of packed weight tiles (+ L2 prefetch)
constexpr int W_MMA = 1;        // tensor memory owner; one elected lane issues the MMAs
constexpr int W_BLOAD = 2;      // TMA loads of activation rows
constexpr int W_EPI = 4;        // warps 4-11: accumulator epilogue, two warps per 32-lane quadrant
constexpr int N_EPI = 8;
constexpr int W_DEQ = 12;       // warps 12-27: Q4 -> bf16 dequantisation, one 16-row tile group each
constexpr int N_DEQ = 16;
constexpr int PF_THREADS = 32 * (W_DEQ + N_DEQ);

struct PfBars {
  uint64_t pk_full[PF_PS], pk_empty[PF_PS];
  uint64_t a_full[PF_SA], a_empty[PF_SA];
  uint64_t b_full[PF_SB], b_empty[PF_SB];
  uint64_t acc_full[2], acc_empty[2], fin;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PfBars) <= 256, "barrier block");
static_assert(PF_SMEM <= 232448, "shared memory");

// Packed weights are read through four TMA tensor maps over the packed
// buffer seen as a 3-D array [tile][k-step][u32]: the codes (128 words = 512
// bytes per tile and k-step) and the scales (32 words = 128 bytes, starting
// cb bytes into each tile), each with a load box of 8 tiles x 1 k-step and an
// L2-prefetch box of 8 tiles x 8 k-steps. Activation rows (B) come through a
// 2-D map [rows][K] bf16 with 64 x 64 boxes in the 128-byte swizzle, which
// is the K-major operand layout the MMA reads.
struct PfGemm {
  CUtensorMap tm_codes, tm_scales, tm_codes_pf, tm_scales_pf, tm_b;
  int tiles_per_expert;      // packed 16-row tiles per expert
  int fb_tiles;              // packed tiles per feature block (A0 tile 0 of block fb = fb * fb_tiles)
  int a1_tiles;              // A1 tile 0 relative to A0 tile 0, in tiles
  int ksteps;                // reduction length / 64
  const int4 *tiles;         // {expert, feature block, first pair in expert, pairs}
  const int32_t *ntiles;
  const int32_t *off, *poff, *ptok;
  const float *pgate;
  __nv_bfloat16 *hout;       // GEMM 1 output, [rows, I]
  int ldh;
  float *y;                  // GEMM 2 output, [T, H] (mode 1) or [pairs, H] in bucket order (mode 2)
  int ldy;
  int mode;                  // 0: silu(G) * U -> h; 1: gate-scaled reduction into y; 2: gate-scaled pair rows
  int32_t *status;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~(uintptr_t)1023);
}

__device__ __forceinline__ bool aborted(PfBars *b) { return *reinterpret_cast<volatile int *>(&b->abort) != 0; }

// Bounded wait on an mbarrier phase. Gives up when another role has aborted,
// or sets the abort flag and the timeout status when the budget runs out.
// sleepy: back off with nanosleep between polls (for waits that last a whole
// tile, so the waiting warps leave issue slots to the ones doing the work).
__device__ __noinline__ bool pf_wait_slow(uint64_t *bar, uint32_t parity, PfBars *b, int32_t *status, bool sleepy) {
  const long long deadline = clock64() + WAIT_BUDGET_CYCLES;
  unsigned ns = 32;
  while (!mbar_try_wait(bar, parity)) {
    if (aborted(b)) return false;
    if (clock64() > deadline) {
      *reinterpret_cast<volatile int *>(&b->abort) = 1;
      set_status(status, DEV_TIMEOUT);
      return false;
    }
    if (sleepy) {
      __nanosleep(ns);
      ns = ns < 1024 ? 2 * ns : 1024;
    }
  }
  return true;
}

__device__ __forceinline__ bool pf_wait(uint64_t *bar, uint32_t parity, PfBars *b, int32_t *status,
                                        bool sleepy = false) {
  if (mbar_try_wait(bar, parity)) return true;
  return pf_wait_slow(bar, parity, b, status, sleepy);
}

// Every lane waits; the warp proceeds only if all lanes saw the phase.
__device__ __forceinline__ bool pf_wait_warp(uint64_t *bar, uint32_t parity, PfBars *b, int32_t *status,
                                             bool sleepy = false) {
  const bool ok = pf_wait(bar, parity, b, status, sleepy);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *m, int x, int y, int z, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *m, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *m, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(m)), "r"(x),
               "r"(y)
               : "memory");
}
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *m, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

__device__ __forceinline__ uint32_t fma_bf16x2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Two 4-bit codes at bits 0-3 and 16-19 -> bf16x2 (128 + q0, 128 + q1):
// 0x4300 is bf16 128.0, whose last mantissa bit is worth 1.
__device__ __forceinline__ uint32_t nib2_bf16x2(uint32_t x) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x000F000Fu), "r"(0x43004300u));
  return r;
}

// fp16 bits -> bf16 (round to nearest even), replicated in both halves.
__device__ __forceinline__ uint32_t h2bf_pair(uint32_t h16) {
  const float f = __half2float(__ushort_as_half((unsigned short)h16));
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(r) : "f"(f));
  return r;
}

constexpr uint32_t BF_ONE2 = 0x3F803F80u;     // (1, 1)
constexpr uint32_t BF_M128_2 = 0xC300C300u;   // (-128, -128)

// One packed Q4 word holds 4 consecutive codes of row R (low nibbles) and of
// row R + 8 (high nibbles). Writes w = d*q + m (bf16, one rounding given the
// bf16 d and m, replicated pairs d0/m0 for row R and d1/m1 for row R + 8) for
// both rows into the swizzled K-major operand.
__device__ __forceinline__ void dq_word(uint32_t word, uint32_t d0, uint32_t m0, uint32_t d1, uint32_t m1,
                                        uint8_t *row_lo, uint8_t *row_hi, int byte_off) {
  const uint32_t p01 = __byte_perm(word, 0, 0x4140);
  const uint32_t p23 = __byte_perm(word, 0, 0x4342);
  const uint32_t q01 = fma_bf16x2(nib2_bf16x2(p01), BF_ONE2, BF_M128_2);
  const uint32_t q23 = fma_bf16x2(nib2_bf16x2(p23), BF_ONE2, BF_M128_2);
  const uint32_t r01 = fma_bf16x2(nib2_bf16x2(p01 >> 4), BF_ONE2, BF_M128_2);
  const uint32_t r23 = fma_bf16x2(nib2_bf16x2(p23 >> 4), BF_ONE2, BF_M128_2);
  *reinterpret_cast<uint2 *>(row_lo + byte_off) = make_uint2(fma_bf16x2(q01, d0, m0), fma_bf16x2(q23, d0, m0));
  *reinterpret_cast<uint2 *>(row_hi + byte_off) = make_uint2(fma_bf16x2(r01, d1, m1), fma_bf16x2(r23, d1, m1));
}

// ------------------------------------------------------------------ roles --
// Global index of a tile's A0 tile 0 in the packed buffer's tile array.
__device__ __forceinline__ int pf_z0(const PfGemm &a, int4 t) { return t.x * a.tiles_per_expert + t.y * a.fb_tiles; }

// Makes sure no TMA copy of the last phases issued on a ring is still writing
// shared memory when the CTA exits (bounded; independent of aborts).
__device__ void pf_drain(uint64_t *full, int stages, uint32_t issued, int32_t *status) {
  const uint32_t first = issued > (uint32_t)stages ? issued - stages : 0;
  for (uint32_t u = first; u < issued; ++u)
    if (!mbar_wait(&full[u % stages], (u / stages) & 1, clock64() + WAIT_BUDGET_CYCLES)) set_status(status, DEV_TIMEOUT);
}

// One lane: per k-step four TMA loads (A0/A1 codes, A0/A1 scales, 8 tiles
// each) into a packed stage, and L2 prefetches of the packed weights running
// PF_PREFETCH k-steps ahead (across tiles).
__device__ void pf_producer(const PfGemm &a, uint8_t *sm, PfBars *b, int nt) {
  uint32_t g = 0;
  int pt = blockIdx.x, pks = 0;   // prefetch cursor
  uint32_t pg = 0;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int z0 = pf_z0(a, a.tiles[ti]);
    bool ok = true;
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      while (pg < g + PF_PREFETCH && pt < nt) {
        const int pz = pf_z0(a, a.tiles[pt]);
        tma_prefetch_3d(&a.tm_codes_pf, 0, pks, pz);
        tma_prefetch_3d(&a.tm_codes_pf, 0, pks, pz + a.a1_tiles);
        tma_prefetch_3d(&a.tm_scales_pf, 0, pks, pz);
        tma_prefetch_3d(&a.tm_scales_pf, 0, pks, pz + a.a1_tiles);
        const int n = min(PF_PF_BOX, a.ksteps - pks);
        pks += n;
        pg += n;
        if (pks == a.ksteps) {
          pks = 0;
          pt += gridDim.x;
        }
      }
      const int ps = g % PF_PS;
      if (!pf_wait(&b->pk_empty[ps], ((g / PF_PS) & 1) ^ 1, b, a.status, true)) {
        ok = false;
        break;
      }
      uint8_t *pk = sm + PF_OFF_PK + ps * PF_PK;
      mbar_arrive_expect_tx(&b->pk_full[ps], PF_PK);
      tma_load_3d(pk, &a.tm_codes, 0, s, z0, &b->pk_full[ps]);
      tma_load_3d(pk + 8 * 512, &a.tm_codes, 0, s, z0 + a.a1_tiles, &b->pk_full[ps]);
      tma_load_3d(pk + PF_PK_CODES, &a.tm_scales, 0, s, z0, &b->pk_full[ps]);
      tma_load_3d(pk + PF_PK_CODES + 8 * 128, &a.tm_scales, 0, s, z0 + a.a1_tiles, &b->pk_full[ps]);
    }
    if (!ok) break;
  }
  pf_drain(b->pk_full, PF_PS, g, a.status);
}

// One lane: per k-step ceil(N / 64) TMA loads of 64 activation rows x 64 bf16.
// Rows past the tile (or past the matrix: zero fill) are loaded and not used.
// The same rows' k-step s + PF_B_PREFETCH is prefetched into L2 (64 x 64 boxes).
__device__ void pf_bloader(const PfGemm &a, uint8_t *sm, PfBars *b, int nt) {
  uint32_t g = 0;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int4 t = a.tiles[ti];
    const int N = (t.w + 15) & ~15;
    const int nbox = (N + PF_B_BOX - 1) / PF_B_BOX;
    const int row0 = a.poff[t.x] + t.z;
    for (int s = 0; s < min(PF_B_PREFETCH, a.ksteps); ++s)
      for (int j = 0; j < nbox; ++j) tma_prefetch_2d(&a.tm_b, s * PF_KS, row0 + j * PF_B_BOX);
    bool ok = true;
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      if (s + PF_B_PREFETCH < a.ksteps)
        for (int j = 0; j < nbox; ++j) tma_prefetch_2d(&a.tm_b, (s + PF_B_PREFETCH) * PF_KS, row0 + j * PF_B_BOX);
      const int st = g % PF_SB;
      if (!pf_wait(&b->b_empty[st], ((g / PF_SB) & 1) ^ 1, b, a.status, true)) {
        ok = false;
        break;
      }
      uint8_t *B = sm + PF_OFF_B + st * PF_B_BYTES;
      mbar_arrive_expect_tx(&b->b_full[st], nbox * PF_B_BOX * PF_KS * 2);
      for (int j = 0; j < nbox; ++j)
        tma_load_2d(B + j * PF_B_BOX * 128, &a.tm_b, s * PF_KS, row0 + j * PF_B_BOX, &b->b_full[st]);
    }
    if (!ok) break;
  }
  pf_drain(b->b_full, PF_SB, g, a.status);
}

__device__ void pf_dequant(const PfGemm &a, uint8_t *sm, PfBars *b, int nt) {
  const int w = (threadIdx.x >> 5) - W_DEQ;     // tile group: A0 tiles 0-7, then A1 tiles 0-7
  const int lane = threadIdx.x & 31, g8 = lane >> 2, t4 = lane & 3;
  const int half = w >> 3, tile = w & 7;
  const int sub = (t4 & 1) * 8, cb = t4 >> 1;
  uint32_t g = 0;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      const int ps = g % PF_PS, st = g % PF_SA;
      if (!pf_wait_warp(&b->pk_full[ps], (g / PF_PS) & 1, b, a.status)) return;
      const uint8_t *pk = sm + PF_OFF_PK + ps * PF_PK;
      const uint4 c = *reinterpret_cast<const uint4 *>(pk + w * 512 + lane * 16);
      const uint32_t *sc = reinterpret_cast<const uint32_t *>(pk + PF_PK_CODES + w * 128);
      const uint2 s0 = *reinterpret_cast<const uint2 *>(sc + g8 * 2);        // block 0: rows g8, g8+8
      const uint2 s1 = *reinterpret_cast<const uint2 *>(sc + 16 + g8 * 2);   // block 1
      __syncwarp();
      if (lane == 0) mbar_arrive(&b->pk_empty[ps]);
      const uint32_t d00 = h2bf_pair(s0.x & 0xFFFFu), m00 = h2bf_pair(s0.x >> 16);
      const uint32_t d01 = h2bf_pair(s0.y & 0xFFFFu), m01 = h2bf_pair(s0.y >> 16);
      const uint32_t d10 = h2bf_pair(s1.x & 0xFFFFu), m10 = h2bf_pair(s1.x >> 16);
      const uint32_t d11 = h2bf_pair(s1.y & 0xFFFFu), m11 = h2bf_pair(s1.y >> 16);
      if (!pf_wait_warp(&b->a_empty[st], ((g / PF_SA) & 1) ^ 1, b, a.status)) return;
      uint8_t *row_lo = sm + st * PF_ASTAGE + half * PF_A_BYTES + (16 * tile + g8) * 128;
      uint8_t *row_hi = row_lo + 8 * 128;
      // word q: block q/2, codes k = 32*(q/2) + 16*(q%2) + 4*t4 + i; 16-byte
      // chunk (k/8) swizzled by the row's position in its 8-row group (g8)
      dq_word(c.x, d00, m00, d01, m01, row_lo, row_hi, (((0 + cb) ^ g8) << 4) + sub);
      dq_word(c.y, d00, m00, d01, m01, row_lo, row_hi, (((2 + cb) ^ g8) << 4) + sub);
      dq_word(c.z, d10, m10, d11, m11, row_lo, row_hi, (((4 + cb) ^ g8) << 4) + sub);
      dq_word(c.w, d10, m10, d11, m11, row_lo, row_hi, (((6 + cb) ^ g8) << 4) + sub);
      tc05::fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b->a_full[st]);
    }
  }
}

// Accumulator slots, walked the same way by the MMA warp and the epilogue
// warps: a narrow tile (at most PF_NARROW tokens) takes the next slot, its
// second accumulator PF_NARROW columns after the first; a wide tile takes both
// slots, its second accumulator in slot 1. use[s] counts the tiles that took
// slot s, which gives the phase of that slot's barriers.
struct AccSlots {
  uint32_t use[2] = {0, 0};
  int next = 0;
  int first, second_off;   // of the current tile
  bool wide;
  __device__ void take(int tokens) {
    wide = tokens > PF_NARROW;
    first = wide ? 0 : next;
    second_off = wide ? PF_SLOT : PF_NARROW;
  }
  __device__ void done() {
    ++use[first];
    if (wide) ++use[1];
    next = wide ? 0 : first ^ 1;
  }
};

// The whole warp runs the loop (waits, descriptor arithmetic) so every value
// stays warp-uniform; one elected lane issues the tensor-core instructions.
// Issuing from a lone lane in a divergent branch measured about 2.5x slower
// per MMA, which made the issue loop the limit for small tiles.
__device__ void pf_mma(const PfGemm &a, uint8_t *sm, PfBars *b, int nt, uint32_t tmem) {
  const uint32_t base = smem_u32(sm);
  // descriptors of stage 0; a stage's start address is added in 16-byte units
  const uint64_t da0 = tc05::sw128_desc(base), db0 = tc05::sw128_desc(base + PF_OFF_B);
  uint32_t g = 0;
  AccSlots sl;
  bool issued = false;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int4 t = a.tiles[ti];
    const uint32_t idesc = tc05::idesc_bf16_f32(PF_M, (t.w + 15) & ~15);
    sl.take(t.w);
    const uint32_t acc0 = tmem + sl.first * PF_SLOT, acc1 = acc0 + sl.second_off;
    if (!pf_wait_warp(&b->acc_empty[sl.first], (sl.use[sl.first] & 1) ^ 1, b, a.status)) goto done;
    if (sl.wide && !pf_wait_warp(&b->acc_empty[1], (sl.use[1] & 1) ^ 1, b, a.status)) goto done;
    tc05::fence_after_sync();
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      const int sa = g % PF_SA, sb = g % PF_SB;
      if (!pf_wait_warp(&b->a_full[sa], (g / PF_SA) & 1, b, a.status)) goto done;
      if (!pf_wait_warp(&b->b_full[sb], (g / PF_SB) & 1, b, a.status)) goto done;
      tc05::fence_after_sync();
      issued = true;
      const uint64_t d0 = da0 + (uint64_t)(sa * (PF_ASTAGE >> 4)), d1 = d0 + (PF_A_BYTES >> 4);
      const uint64_t db = db0 + (uint64_t)(sb * (PF_B_BYTES >> 4));
      if (tc05::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < PF_KS / 16; ++kk) {
          const uint32_t acc = (s | kk) != 0;
          tc05::mma_bf16(acc0, d0 + 2 * kk, db + 2 * kk, idesc, acc);
          tc05::mma_bf16(acc1, d1 + 2 * kk, db + 2 * kk, idesc, acc);
        }
        tc05::commit(&b->a_empty[sa]);
        tc05::commit(&b->b_empty[sb]);
      }
      __syncwarp();
    }
    if (tc05::elect_one()) {
      tc05::commit(&b->acc_full[sl.first]);
      if (sl.wide) tc05::commit(&b->acc_full[1]);
    }
    __syncwarp();
    sl.done();
  }
done:
  // every MMA the issuing lane (lane 0: the lowest lane of the converged
  // warp) issued has completed before tensor memory is freed
  if (issued && (threadIdx.x & 31) == 0) {
    tc05::commit(&b->fin);
    if (!mbar_wait(&b->fin, 0, clock64() + WAIT_BUDGET_CYCLES)) set_status(a.status, DEV_TIMEOUT);
  }
  __syncwarp();
}

__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// Epilogue warp pair (q, q + 4) shares TMEM lane quadrant q and alternates
// 16-column chunks.
__device__ void pf_epilogue(const PfGemm &a, PfBars *b, int nt, uint32_t tmem) {
  const int ew = (threadIdx.x >> 5) - W_EPI;
  const int q = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31, par = ew >> 2;
  const int r = 32 * q + lane;
  const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
  AccSlots sl;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int4 t = a.tiles[ti];
    const int N = (t.w + 15) & ~15;
    sl.take(t.w);
    const uint32_t ts = tq + sl.first * PF_SLOT, tu = ts + sl.second_off;
    if (!pf_wait_warp(&b->acc_full[sl.first], sl.use[sl.first] & 1, b, a.status, true)) return;
    if (sl.wide && !pf_wait_warp(&b->acc_full[1], sl.use[1] & 1, b, a.status, true)) return;
    tc05::fence_after_sync();
    if (a.mode == 0) {
      __nv_bfloat16 *h = a.hout + (size_t)(a.poff[t.x] + t.z) * a.ldh + t.y * PF_M + r;
      for (int c0 = 16 * par; c0 < N; c0 += 32) {
        float gv[16], uv[16];
        tc05::ld16x2(ts + c0, tu + c0, gv, uv);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // lanes 2m and 2m+1 hold adjacent features: even lanes store the pair
          const int n = c0 + i;
          const float hv = n < t.w ? silu(gv[i]) * uv[i] : 0.0f;
          const float hn = __shfl_down_sync(0xffffffffu, hv, 1);
          if (!(lane & 1))
            *reinterpret_cast<__nv_bfloat162 *>(h + (size_t)n * a.ldh) = __floats2bfloat162_rn(hv, hn);
        }
      }
    } else if (a.mode == 2) {
      const int pos0 = a.off[t.x] + t.z;
      float *pb = a.y + (size_t)pos0 * a.ldy + t.y * (2 * PF_M) + r;
      for (int c0 = 16 * par; c0 < N; c0 += 32) {
        float v0[16], v1[16];
        tc05::ld16x2(ts + c0, tu + c0, v0, v1);
        float gt = 0.0f;
        if (lane < 16 && c0 + lane < t.w) gt = a.pgate[pos0 + c0 + lane];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float gi = __shfl_sync(0xffffffffu, gt, i);
          if (c0 + i < t.w) {
            float *pr = pb + (size_t)(c0 + i) * a.ldy;
            pr[0] = __fmul_rn(gi, v0[i]);
            pr[PF_M] = __fmul_rn(gi, v1[i]);
          }
        }
      }
    } else {
      const int pos0 = a.off[t.x] + t.z;
      float *yb = a.y + t.y * (2 * PF_M) + r;
      for (int c0 = 16 * par; c0 < N; c0 += 32) {
        float v0[16], v1[16];
        tc05::ld16x2(ts + c0, tu + c0, v0, v1);
        // lane i < 16 fetches column c0 + i's token and gate; shuffles broadcast them
        int tk = 0;
        float gt = 0.0f;
        if (lane < 16 && c0 + lane < t.w) {
          tk = a.ptok[pos0 + c0 + lane];
          gt = a.pgate[pos0 + c0 + lane];
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int tok = __shfl_sync(0xffffffffu, tk, i);
          const float gi = __shfl_sync(0xffffffffu, gt, i);
          if (c0 + i < t.w) {
            float *yr = yb + (size_t)tok * a.ldy;
            atomicAdd(yr, gi * v0[i]);
            atomicAdd(yr + PF_M, gi * v1[i]);
          }
        }
      }
    }
    tc05::fence_before_sync();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&b->acc_empty[sl.first]);
      if (sl.wide) mbar_arrive(&b->acc_empty[1]);
    }
    sl.done();
  }
}

__global__ void __launch_bounds__(PF_THREADS, 1) pf_gemm_kernel(const __grid_constant__ PfGemm a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  PfBars *b = reinterpret_cast<PfBars *>(sm + PF_OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < PF_PS; ++i) {
      mbar_init(&b->pk_full[i], 1);
      mbar_init(&b->pk_empty[i], N_DEQ);
    }
    for (int i = 0; i < PF_SA; ++i) {
      mbar_init(&b->a_full[i], N_DEQ);
      mbar_init(&b->a_empty[i], 1);
    }
    for (int i = 0; i < PF_SB; ++i) {
      mbar_init(&b->b_full[i], 1);
      mbar_init(&b->b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b->acc_full[i], 1);
      mbar_init(&b->acc_empty[i], N_EPI);
    }
    mbar_init(&b->fin, 1);
    b->abort = 0;
    fence_mbar_init();
  }
  if (warp == W_MMA) {
    tc05::tmem_alloc(&b->tmem_base, PF_TMEM_COLS);
    tc05::tmem_relinquish();
  }
  if (threadIdx.x == 32 * W_PRODUCER) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tm_codes)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tm_scales)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tm_b)) : "memory");
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = b->tmem_base;
  const int nt = *a.ntiles;

  if (warp == W_PRODUCER) {
    if (lane == 0) pf_producer(a, sm, b, nt);
    __syncwarp();
  } else if (warp == W_MMA) {
    pf_mma(a, sm, b, nt, tmem);
  } else if (warp == W_BLOAD) {
    if (lane == 0) pf_bloader(a, sm, b, nt);
    __syncwarp();
  } else if (warp >= W_EPI && warp < W_EPI + N_EPI) {
    pf_epilogue(a, b, nt, tmem);
  } else if (warp >= W_DEQ) {
    pf_dequant(a, sm, b, nt);
  }

  tc05::fence_before_sync();
  __syncthreads();
  if (warp == W_MMA) {
    tc05::fence_after_sync();
    tc05::tmem_dealloc(tmem, PF_TMEM_COLS);
  }
}

// -------------------------------------------------------- activation gather --
// Xp[row] = x[token of the row's pair] for every padded bucket row, zero in
// each expert's padding rows. One warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) pf_gather_kernel(const uint4 *__restrict__ x, int H8, const int32_t *off,
                                                        const int32_t *poff, const int32_t *ptok, int E, int rows,
                                                        uint4 *__restrict__ xp, const int32_t *status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows || *reinterpret_cast<volatile const int32_t *>(status) != 0) return;
  if (row >= poff[E]) return;
  int lo = 0, hi = E;   // largest e with poff[e] <= row
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (poff[mid] <= row) lo = mid;
    else hi = mid;
  }
  const int i = row - poff[lo];
  uint4 *dst = xp + (size_t)row * H8;
  if (i < off[lo + 1] - off[lo]) {
    const uint4 *src = x + (size_t)ptok[off[lo] + i] * H8;
    for (int c = lane; c < H8; c += 32) dst[c] = src[c];
  } else {
    for (int c = lane; c < H8; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
  }
}

// ------------------------------------------------------------- tile plan --
struct PlanArgs {
  const int32_t *off;   // [E + 1] bucket offsets
  int E, fbs1, fbs2;
  int32_t *poff;        // [E + 1] padded row offsets of h
  int4 *tiles1, *tiles2;
  int32_t *ntiles;      // [2]
  const int32_t *status;
};

// Tiles of at most PF_N pairs per expert: the full PF_N-pair chunks first, in
// (expert, chunk, feature block) order, then each expert's remainder chunk,
// largest remainder first (ties by expert index), all feature blocks of one
// remainder adjacent. CTAs take tiles round-robin.
// Position of every pair (t, j) in bucket order: inv[perm[i]] = i.
__global__ void pf_inverse_kernel(const int32_t *perm, int P, int32_t *inv, const int32_t *status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < P && *reinterpret_cast<volatile const int32_t *>(status) == 0) inv[perm[i]] = i;
}

// y[t, :] = sum_j part[inv[t k + j], :] in slot order, one rounding per add.
// One thread per 4 features of a token; H4 = H / 4.
__global__ void __launch_bounds__(256) pf_combine_kernel(const float4 *part, const int32_t *inv, int T, int k, int H4,
                                                         float4 *y, const int32_t *status) {
  const long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= (long long)T * H4 || *reinterpret_cast<volatile const int32_t *>(status) != 0) return;
  const int t = (int)(o / H4), c = (int)(o % H4);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float4 v = __ldg(part + (size_t)inv[t * k + j] * H4 + c);
    acc.x = __fadd_rn(acc.x, v.x);
    acc.y = __fadd_rn(acc.y, v.y);
    acc.z = __fadd_rn(acc.z, v.z);
    acc.w = __fadd_rn(acc.w, v.w);
  }
  y[o] = acc;
}

__global__ void __launch_bounds__(1024, 1) pf_plan_kernel(PlanArgs a) {
  __shared__ int s_rem[PF_MAX_E];
  __shared__ int wt[3][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, E = a.E;
  if (*reinterpret_cast<volatile const int32_t *>(a.status) != 0) {
    if (tid == 0) a.ntiles[0] = a.ntiles[1] = 0;
    return;
  }
  int nfull[2], rem[2], pad[2];
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    const int n = e < E ? a.off[e + 1] - a.off[e] : 0;
    nfull[r] = n / PF_N;
    rem[r] = n % PF_N;
    pad[r] = (n + 15) & ~15;
    if (e < E) s_rem[e] = rem[r];
  }
  const int F = nfull[0] + nfull[1], Q = (rem[0] > 0) + (rem[1] > 0), D = pad[0] + pad[1];
  int iF = F, iQ = Q, iD = D;
  warp_scan3(iF, iQ, iD);
  if (lane == 31) {
    wt[0][warp] = iF;
    wt[1][warp] = iQ;
    wt[2][warp] = iD;
  }
  __syncthreads();
  if (warp == 0) {
    int a0 = wt[0][lane], a1 = wt[1][lane], a2 = wt[2][lane];
    int b0 = a0, b1 = a1, b2 = a2;
    warp_scan3(b0, b1, b2);
    wt[0][lane] = b0 - a0;
    wt[1][lane] = b1 - a1;
    wt[2][lane] = b2 - a2;
  }
  __syncthreads();
  int Fx = wt[0][warp] + iF - F, Dx = wt[2][warp] + iD - D;
  __shared__ int tot_sh[2];
  if (tid == 1023) {   // the last thread's inclusive prefixes are the totals
    tot_sh[0] = Fx + F;
    tot_sh[1] = wt[1][warp] + iQ;
  }
  __syncthreads();
  const int Fall = tot_sh[0], Qall = tot_sh[1];
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    if (e >= E) break;
    a.poff[e] = Dx;
    Dx += pad[r];
    if (e == E - 1) a.poff[E] = Dx;
    for (int c = 0; c < nfull[r]; ++c)
      for (int fb = 0; fb < a.fbs1; ++fb)
        a.tiles1[(size_t)a.fbs1 * (Fx + c) + fb] = make_int4(e, fb, c * PF_N, PF_N);
    for (int c = 0; c < nfull[r]; ++c)
      for (int fb = 0; fb < a.fbs2; ++fb)
        a.tiles2[(size_t)a.fbs2 * (Fx + c) + fb] = make_int4(e, fb, c * PF_N, PF_N);
    Fx += nfull[r];
    if (rem[r] > 0) {
      int rank = 0;
      for (int e2 = 0; e2 < E; ++e2) {
        const int r2 = s_rem[e2];
        rank += (r2 > rem[r] || (r2 == rem[r] && e2 < e)) ? 1 : 0;
      }
      for (int fb = 0; fb < a.fbs1; ++fb)
        a.tiles1[(size_t)a.fbs1 * (Fall + rank) + fb] = make_int4(e, fb, nfull[r] * PF_N, rem[r]);
      for (int fb = 0; fb < a.fbs2; ++fb)
        a.tiles2[(size_t)a.fbs2 * (Fall + rank) + fb] = make_int4(e, fb, nfull[r] * PF_N, rem[r]);
    }
  }
  if (tid == 0) {
    a.ntiles[0] = a.fbs1 * (Fall + Qall);
    a.ntiles[1] = a.fbs2 * (Fall + Qall);
  }
}

// ------------------------------------------------------------ workspace --
struct PfLayout {
  size_t off, poff, perm, ptok, pgate, ntiles, bk, tiles1, tiles2, h, xp, inv, part, total;
  size_t max_tiles1, max_tiles2, h_rows;
};

inline size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

PfLayout pf_layout(int T, int k, int E, int H, int I) {
  PfLayout L{};
  const size_t P = (size_t)T * k;
  const size_t chunks = (P + PF_N - 1) / PF_N + (size_t)E;
  L.max_tiles1 = (size_t)(I / PF_M) * chunks;
  L.max_tiles2 = (size_t)(H / (2 * PF_M)) * chunks;
  L.h_rows = P + 15 * (size_t)E;
  size_t o = 0;
  L.off = o;    o += up256((E + 1) * sizeof(int32_t));
  L.poff = o;   o += up256((E + 1) * sizeof(int32_t));
  L.perm = o;   o += up256(P * sizeof(int32_t));
  L.ptok = o;   o += up256(P * sizeof(int32_t));
  L.pgate = o;  o += up256(P * sizeof(float));
  L.ntiles = o; o += 256;
  L.bk = o;     o += bucket_ws_bytes(T, k, E);
  L.tiles1 = o; o += up256(L.max_tiles1 * sizeof(int4));
  L.tiles2 = o; o += up256(L.max_tiles2 * sizeof(int4));
  L.h = o;      o += up256(L.h_rows * I * sizeof(__nv_bfloat16));
  L.xp = o;     o += up256(L.h_rows * H * sizeof(__nv_bfloat16));
  L.inv = o;    o += up256(P * sizeof(int32_t));
  L.part = o;   o += up256(P * H * sizeof(float));
  L.total = o;
  return L;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D u32 tensor [ntiles][ksteps][inner] at base (tile stride tb bytes, k-step
// stride inner * 4 bytes), box [bt][bk][inner].
bool encode_packed_map(CUtensorMap *m, const void *base, int inner, int ksteps, uint64_t ntiles, uint64_t tb, int bk,
                       int bt) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)ksteps, ntiles};
  const cuuint64_t strides[2] = {(cuuint64_t)inner * 4, tb};
  const cuuint32_t box[3] = {(cuuint32_t)inner, (cuuint32_t)bk, (cuuint32_t)bt};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor [rows][K] (row-major), 64 x 64 boxes in the 128-byte swizzle.
bool encode_rows_map(CUtensorMap *m, const void *base, int K, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)PF_KS, (cuuint32_t)PF_B_BOX};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps over one layer's packed matrix of kind gate_up (K = H) or down (K = I).
bool pf_maps(PfGemm &g, const void *w, int E, int tiles_per_expert, int K) {
  const int bits = QMOE_Q4;
  const uint64_t tb = (uint64_t)tile_bytes(bits, K), cb = (uint64_t)tile_code_bytes(bits, K);
  const uint64_t nt = (uint64_t)E * tiles_per_expert;
  const int ks = K / PF_KS;
  const uint8_t *base = static_cast<const uint8_t *>(w);
  return encode_packed_map(&g.tm_codes, base, 128, ks, nt, tb, 1, 8) &&
         encode_packed_map(&g.tm_scales, base + cb, 32, ks, nt, tb, 1, 8) &&
         encode_packed_map(&g.tm_codes_pf, base, 128, ks, nt, tb, PF_PF_BOX, 8) &&
         encode_packed_map(&g.tm_scales_pf, base + cb, 32, ks, nt, tb, PF_PF_BOX, 8);
}

qmoe_status pf_gemm_launch(const PfGemm &g, cudaStream_t s) {
  if (cudaFuncSetAttribute(pf_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM) != cudaSuccess)
    return QMOE_ERR_CUDA;
  pf_gemm_kernel<<<num_sms(), PF_THREADS, PF_SMEM, s>>>(g);
  note_launch();
  return cuda_status(cudaGetLastError());
}

}  // namespace
}  // namespace qmoe

using namespace qmoe;

extern "C" size_t qmoe_prefill_workspace_bytes(int T, int k, int E, int H, int I) {
  if (T < 1 || k < 1 || E < 1 || H < 1 || I < 1) return 0;
  return pf_layout(T, k, E, H, I).total;
}

static qmoe_status ffn_prefill(const qmoe_experts *ex, const void *x, int T, const int32_t *idx, const float *gate,
                               int k, float *y, void *workspace, size_t workspace_bytes, int32_t *dev_status,
                               qmoe_stream_t stream, void *const *events, int flags) {
  const bool atomic_combine = (flags & QMOE_PREFILL_ATOMIC_COMBINE) != 0;
  if (!ex || !x || !idx || !gate || !y || !workspace || !dev_status) return QMOE_ERR_INVALID_ARG;
  if (T < 1 || k < 1) return QMOE_ERR_INVALID_ARG;
  const int E = ex->E, H = ex->H, I = ex->I;
  if (E < 1 || H < 1 || I < 1 || !ex->gate_up || !ex->down) return QMOE_ERR_INVALID_ARG;
  if (ex->gate_up_bytes != qmoe_packed_bytes(ex->fmt, QMOE_GATE_UP, E, H, I) ||
      ex->down_bytes != qmoe_packed_bytes(ex->fmt, QMOE_DOWN, E, H, I))
    return QMOE_ERR_GEOMETRY;
  if (ex->fmt != QMOE_Q4) return QMOE_ERR_UNSUPPORTED;
  if (H % (2 * PF_M) || I % PF_M || k > E || E > PF_MAX_E) return QMOE_ERR_UNSUPPORTED;
  if ((long long)T * k > (1LL << 28)) return QMOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace) || !aligned16(ex->gate_up) || !aligned16(ex->down))
    return QMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(gate) |
       reinterpret_cast<uintptr_t>(dev_status)) & 3)
    return QMOE_ERR_INVALID_ARG;
  const PfLayout L = pf_layout(T, k, E, H, I);
  if (workspace_bytes < L.total) return QMOE_ERR_WORKSPACE;
  if (!bucket_supported(T, k, E) || (size_t)PF_SMEM > max_smem_optin()) return QMOE_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  char *ws = static_cast<char *>(workspace);
  int32_t *off = reinterpret_cast<int32_t *>(ws + L.off);
  int32_t *poff = reinterpret_cast<int32_t *>(ws + L.poff);
  int32_t *perm = reinterpret_cast<int32_t *>(ws + L.perm);
  int32_t *ptok = reinterpret_cast<int32_t *>(ws + L.ptok);
  float *pgate = reinterpret_cast<float *>(ws + L.pgate);
  int32_t *ntiles = reinterpret_cast<int32_t *>(ws + L.ntiles);
  int4 *tiles1 = reinterpret_cast<int4 *>(ws + L.tiles1);
  int4 *tiles2 = reinterpret_cast<int4 *>(ws + L.tiles2);
  __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(ws + L.h);
  __nv_bfloat16 *xp = reinterpret_cast<__nv_bfloat16 *>(ws + L.xp);

  qmoe_status st = bucket_launch(idx, gate, T, k, E, ws + L.bk, off, perm, ptok, pgate, nullptr, nullptr, true, dev_status, s);
  if (st != QMOE_OK) return st;
  PlanArgs pa{off, E, I / PF_M, H / (2 * PF_M), poff, tiles1, tiles2, ntiles, dev_status};
  pf_plan_kernel<<<1, 1024, 0, s>>>(pa);
  note_launch();
  if (cudaGetLastError() != cudaSuccess) return QMOE_ERR_CUDA;
  int32_t *inv = reinterpret_cast<int32_t *>(ws + L.inv);
  float *part = reinterpret_cast<float *>(ws + L.part);
  const int P = T * k;
  if (atomic_combine) {
    if (cudaMemsetAsync(y, 0, (size_t)T * H * sizeof(float), s) != cudaSuccess) return QMOE_ERR_CUDA;
  } else {
    pf_inverse_kernel<<<(P + 255) / 256, 256, 0, s>>>(perm, P, inv, dev_status);
    note_launch();
    if (cudaGetLastError() != cudaSuccess) return QMOE_ERR_CUDA;
  }
  pf_gather_kernel<<<(unsigned)((L.h_rows + 7) / 8), 256, 0, s>>>(static_cast<const uint4 *>(x), H / 8, off, poff, ptok,
                                                                   E, (int)L.h_rows, reinterpret_cast<uint4 *>(xp),
                                                                   dev_status);
  note_launch();
  if (cudaGetLastError() != cudaSuccess) return QMOE_ERR_CUDA;

  PfGemm g1{};
  g1.tiles_per_expert = 2 * (I / 16);
  if (!pf_maps(g1, ex->gate_up, E, g1.tiles_per_expert, H)) return QMOE_ERR_CUDA;
  g1.fb_tiles = PF_M / 16;
  g1.a1_tiles = I / 16;
  g1.ksteps = H / PF_KS;
  if (!encode_rows_map(&g1.tm_b, xp, H, L.h_rows)) return QMOE_ERR_CUDA;
  g1.tiles = tiles1;
  g1.ntiles = ntiles;
  g1.off = off;
  g1.poff = poff;
  g1.ptok = ptok;
  g1.pgate = pgate;
  g1.hout = h;
  g1.ldh = I;
  g1.mode = 0;
  g1.status = dev_status;
  if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[0]), s) != cudaSuccess) return QMOE_ERR_CUDA;
  st = pf_gemm_launch(g1, s);
  if (st != QMOE_OK) return st;
  if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[1]), s) != cudaSuccess) return QMOE_ERR_CUDA;

  PfGemm g2 = g1;
  g2.tiles_per_expert = H / 16;
  if (!pf_maps(g2, ex->down, E, g2.tiles_per_expert, I)) return QMOE_ERR_CUDA;
  g2.fb_tiles = 2 * PF_M / 16;
  g2.a1_tiles = PF_M / 16;
  g2.ksteps = I / PF_KS;
  if (!encode_rows_map(&g2.tm_b, h, I, L.h_rows)) return QMOE_ERR_CUDA;
  g2.tiles = tiles2;
  g2.ntiles = ntiles + 1;
  g2.hout = nullptr;
  g2.y = atomic_combine ? y : part;
  g2.ldy = H;
  g2.mode = atomic_combine ? 1 : 2;
  st = pf_gemm_launch(g2, s);
  if (st != QMOE_OK) return st;
  if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[2]), s) != cudaSuccess) return QMOE_ERR_CUDA;
  if (!atomic_combine) {
    const long long n = (long long)T * (H / 4);
    pf_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(reinterpret_cast<const float4 *>(part), inv, T, k,
                                                                 H / 4, reinterpret_cast<float4 *>(y), dev_status);
    note_launch();
    if (cudaGetLastError() != cudaSuccess) return QMOE_ERR_CUDA;
  }
  return QMOE_OK;
}

extern "C" qmoe_status qmoe_ffn_prefill(const qmoe_experts *ex, const void *x, int T, const int32_t *idx,
                                        const float *gate, int k, float *y, void *workspace, size_t workspace_bytes,
                                        int32_t *dev_status, qmoe_stream_t stream) {
  return ffn_prefill(ex, x, T, idx, gate, k, y, workspace, workspace_bytes, dev_status, stream, nullptr, 0);
}

extern "C" qmoe_status qmoe_ffn_prefill_timed(const qmoe_experts *ex, const void *x, int T, const int32_t *idx,
                                              const float *gate, int k, float *y, void *workspace,
                                              size_t workspace_bytes, int32_t *dev_status, qmoe_stream_t stream,
                                              void *const *events, int flags) {
  if (!events || !events[0] || !events[1] || !events[2]) return QMOE_ERR_INVALID_ARG;
  if (flags & ~QMOE_PREFILL_ATOMIC_COMBINE) return QMOE_ERR_INVALID_ARG;
  return ffn_prefill(ex, x, T, idx, gate, k, y, workspace, workspace_bytes, dev_status, stream, events, flags);
}
