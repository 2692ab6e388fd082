// Prefill expert FFN for chunks of many tokens ([P3] batched prefill in chunks,
// "Understanding the Architecture"): bucketing of the routed (token, slot)
// pairs by expert, a tile plan, and two grouped GEMMs on the fifth-generation
// tensor cores with the Q4 expert weights dequantised to bf16 in shared memory.
//
//   GEMM 1, per expert e and 128 intermediate features f:
//       G = Wg[f,:] X_e^T,  U = Wu[f,:] X_e^T      (fp32 in tensor memory)
//       h[pair, f] = bf16(silu(G) * U)
//   GEMM 2, per expert e and 256 hidden features o:
//       Y = Wd[o,:] h_e^T;  y[token, o] += gate[pair] * Y   (fp32 reductions)
// X_e is the bf16 activation rows of the tokens routed to e, gathered by
// token id; h is kept in bucket order with every expert's rows padded to a
// multiple of 16. The weights form the 128-row MMA operand and the tokens the
// N operand (16..256, a multiple of 16), so an expert with n tokens costs
// ceil(n/16)*16 columns, not a 128-row tile.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "layout.cuh"
#include "tc05.cuh"

namespace qmoe {

size_t bucket_smem_bytes(int E);
bool bucket_supported(int T, int k, int E);
qmoe_status bucket_launch(const int32_t *idx, const float *gate, int T, int k, int E, int32_t *offsets, int32_t *perm,
                          int32_t *ptok, float *pgate, int32_t *active, int32_t *nactive, bool check_dup,
                          int32_t *status, cudaStream_t s);

namespace {

constexpr int PF_N = 256;                               // max tokens per tile (MMA N)
constexpr int PF_M = 128;                               // rows per A operand (MMA M)
constexpr int PF_KS = 64;                               // reduction elements per pipeline step
constexpr int PF_S = 3;                                 // operand stages (A0, A1, B)
constexpr int PF_PS = 3;                                // packed-weight stages
constexpr int PF_A_BYTES = PF_M * PF_KS * 2;            // 16 KB
constexpr int PF_B_BYTES = PF_N * PF_KS * 2;            // 32 KB
constexpr int PF_STAGE = 2 * PF_A_BYTES + PF_B_BYTES;   // 64 KB
constexpr int PF_PK_CODES = 16 * 512;                   // 16 tile groups x 64 Q4 codes x 16 rows
constexpr int PF_PK_SCALES = 16 * 128;                  // 16 tiles x 2 blocks x 16 rows x (d, m)
constexpr int PF_PK = PF_PK_CODES + PF_PK_SCALES;
constexpr int PF_OFF_PK = PF_S * PF_STAGE;
constexpr int PF_OFF_BAR = PF_OFF_PK + PF_PS * PF_PK;
constexpr int PF_SMEM = PF_OFF_BAR + 256 + 1024;        // barriers + alignment slack
constexpr int PF_THREADS = 512;
constexpr int PF_TMEM_COLS = 512;                       // two fp32 accumulators of up to 256 columns
constexpr int PF_MAX_E = 1024;

// warp roles
constexpr int W_PRODUCER = 0;   // bulk copies of packed weight tiles
constexpr int W_MMA = 1;        // tensor memory owner; lane 0 issues the MMAs
constexpr int W_BLOAD = 2;      // warps 2-3: gathers of activation rows (cp.async)
constexpr int N_BLOAD = 2;
constexpr int W_EPI = 4;        // warps 4-7: accumulator epilogue, one 32-lane quadrant each
constexpr int W_DEQ = 8;        // warps 8-15: Q4 -> bf16 dequantisation
constexpr int N_DEQ = 8;

struct PfBars {
  uint64_t pk_full[PF_PS], pk_empty[PF_PS];
  uint64_t a_full[PF_S], b_full[PF_S], empty[PF_S];
  uint64_t acc_full, acc_empty, fin;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PfBars) <= 256, "barrier block");

struct PfGemm {
  const uint8_t *w;          // packed matrices of all experts of the layer
  size_t w_expert;           // packed bytes per expert
  int tb, cb;                // bytes per packed 16-row tile; code bytes per tile
  int fb_tiles;              // packed tiles per feature block (A0 tile 0 of block fb = fb * fb_tiles)
  int a1_tiles;              // A1 tile 0 relative to A0 tile 0, in tiles
  int ksteps;                // reduction length / 64
  const __nv_bfloat16 *bsrc; // GEMM 1: x [T, H]; GEMM 2: h [rows, I]
  int ldb;
  int gather;                // 1: B rows are tokens (ptok); 0: B rows are padded bucket rows
  const int4 *tiles;         // {expert, feature block, first pair in expert, pairs}
  const int32_t *ntiles;
  const int32_t *off, *poff, *ptok;
  const float *pgate;
  __nv_bfloat16 *hout;       // GEMM 1 output, [rows, I]
  int ldh;
  float *y;                  // GEMM 2 output, [T, H]
  int ldy;
  int mode;                  // 0: silu(G) * U -> h; 1: gate-scaled reduction into y
  int32_t *status;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~(uintptr_t)1023);
}

__device__ __forceinline__ bool aborted(PfBars *b) { return *reinterpret_cast<volatile int *>(&b->abort) != 0; }

// Bounded wait on an mbarrier phase. Gives up when another role has aborted,
// or sets the abort flag and the timeout status when the budget runs out.
__device__ __noinline__ bool pf_wait(uint64_t *bar, uint32_t parity, PfBars *b, int32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long deadline = clock64() + WAIT_BUDGET_CYCLES;
  while (!mbar_try_wait(bar, parity)) {
    if (aborted(b)) return false;
    if (clock64() > deadline) {
      *reinterpret_cast<volatile int *>(&b->abort) = 1;
      set_status(status, DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Every lane waits; the warp proceeds only if all lanes saw the phase.
__device__ __forceinline__ bool pf_wait_warp(uint64_t *bar, uint32_t parity, PfBars *b, int32_t *status) {
  const bool ok = pf_wait(bar, parity, b, status);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

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
  const uint32_t b = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
  return b | (b << 16);
}

constexpr uint32_t BF_ONE2 = 0x3F803F80u;     // (1, 1)
constexpr uint32_t BF_M128_2 = 0xC300C300u;   // (-128, -128)

// One packed Q4 word holds 4 consecutive codes of row R (low nibbles) and of
// row R + 8 (high nibbles). Writes w = d*q + m (bf16, one rounding given the
// bf16 d and m) for both rows into the swizzled K-major operand.
__device__ __forceinline__ void dq_word(uint32_t word, uint32_t dm_lo, uint32_t dm_hi, uint8_t *row_lo,
                                        uint8_t *row_hi, int byte_off) {
  const uint32_t p01 = __byte_perm(word, 0, 0x4140);
  const uint32_t p23 = __byte_perm(word, 0, 0x4342);
  const uint32_t d0 = h2bf_pair(dm_lo & 0xFFFFu), m0 = h2bf_pair(dm_lo >> 16);
  const uint32_t d1 = h2bf_pair(dm_hi & 0xFFFFu), m1 = h2bf_pair(dm_hi >> 16);
  const uint32_t q01 = fma_bf16x2(nib2_bf16x2(p01), BF_ONE2, BF_M128_2);
  const uint32_t q23 = fma_bf16x2(nib2_bf16x2(p23), BF_ONE2, BF_M128_2);
  const uint32_t r01 = fma_bf16x2(nib2_bf16x2(p01 >> 4), BF_ONE2, BF_M128_2);
  const uint32_t r23 = fma_bf16x2(nib2_bf16x2(p23 >> 4), BF_ONE2, BF_M128_2);
  *reinterpret_cast<uint2 *>(row_lo + byte_off) = make_uint2(fma_bf16x2(q01, d0, m0), fma_bf16x2(q23, d0, m0));
  *reinterpret_cast<uint2 *>(row_hi + byte_off) = make_uint2(fma_bf16x2(r01, d1, m1), fma_bf16x2(r23, d1, m1));
}

// ------------------------------------------------------------------ roles --
__device__ void pf_producer(const PfGemm &a, uint8_t *sm, PfBars *b, int nt) {
  const int lane = threadIdx.x & 31;
  const int j = lane & 15;
  uint32_t g = 0;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int4 t = a.tiles[ti];
    const uint8_t *a0 = a.w + (size_t)t.x * a.w_expert + (size_t)t.y * a.fb_tiles * a.tb;
    const uint8_t *tp = a0 + (size_t)(j < 8 ? j : a.a1_tiles + j - 8) * a.tb;
    bool ok = true;
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      const int ps = g % PF_PS;
      if (!pf_wait_warp(&b->pk_empty[ps], ((g / PF_PS) & 1) ^ 1, b, a.status)) {
        ok = false;
        break;
      }
      uint8_t *pk = sm + PF_OFF_PK + ps * PF_PK;
      if (lane == 0) mbar_arrive_expect_tx(&b->pk_full[ps], PF_PK);
      __syncwarp();
      if (lane < 16)
        bulk_g2s(pk + j * 512, tp + (size_t)s * 512, 512, &b->pk_full[ps]);
      else
        bulk_g2s(pk + PF_PK_CODES + j * 128, tp + a.cb + (size_t)s * 128, 128, &b->pk_full[ps]);
    }
    if (!ok) break;
  }
  // No copy may still be writing shared memory when the CTA exits: wait for
  // the last phase issued on every stage (bounded; independent of aborts).
  const uint32_t first = g > PF_PS ? g - PF_PS : 0;
  for (uint32_t u = first; u < g; ++u) {
    if (!mbar_wait(&b->pk_full[u % PF_PS], (u / PF_PS) & 1, clock64() + WAIT_BUDGET_CYCLES))
      set_status(a.status, DEV_TIMEOUT);
  }
}

__device__ void pf_dequant(const PfGemm &a, uint8_t *sm, PfBars *b, int nt) {
  const int w = (threadIdx.x >> 5) - W_DEQ;
  const int lane = threadIdx.x & 31, g8 = lane >> 2, t4 = lane & 3;
  uint32_t g = 0;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      const int ps = g % PF_PS, st = g % PF_S;
      if (!pf_wait_warp(&b->pk_full[ps], (g / PF_PS) & 1, b, a.status)) return;
      if (!pf_wait_warp(&b->empty[st], ((g / PF_S) & 1) ^ 1, b, a.status)) return;
      const uint8_t *pk = sm + PF_OFF_PK + ps * PF_PK;
      uint8_t *stage = sm + st * PF_STAGE;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int jt = w + 8 * half;   // tile group: A0 tile w, then A1 tile w
        const uint4 c = *reinterpret_cast<const uint4 *>(pk + jt * 512 + lane * 16);
        const uint32_t *sc = reinterpret_cast<const uint32_t *>(pk + PF_PK_CODES + jt * 128);
        const uint2 s0 = *reinterpret_cast<const uint2 *>(sc + g8 * 2);        // block 0: rows g8, g8+8
        const uint2 s1 = *reinterpret_cast<const uint2 *>(sc + 16 + g8 * 2);   // block 1
        uint8_t *row_lo = stage + half * PF_A_BYTES + (16 * w + g8) * 128;
        uint8_t *row_hi = row_lo + 8 * 128;
        // word q: block q/2, codes k = 32*(q/2) + 16*(q%2) + 4*t4 + i; 16-byte
        // chunk (k/8) swizzled by the row's position in its 8-row group (g8)
        const int sub = (t4 & 1) * 8, cb = t4 >> 1;
        dq_word(c.x, s0.x, s0.y, row_lo, row_hi, (((0 + cb) ^ g8) << 4) + sub);
        dq_word(c.y, s0.x, s0.y, row_lo, row_hi, (((2 + cb) ^ g8) << 4) + sub);
        dq_word(c.z, s1.x, s1.y, row_lo, row_hi, (((4 + cb) ^ g8) << 4) + sub);
        dq_word(c.w, s1.x, s1.y, row_lo, row_hi, (((6 + cb) ^ g8) << 4) + sub);
      }
      tc05::fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&b->pk_empty[ps]);
        mbar_arrive(&b->a_full[st]);
      }
    }
  }
}

__device__ void pf_bload(const PfGemm &a, uint8_t *sm, PfBars *b, int nt) {
  const int tid = threadIdx.x - W_BLOAD * 32;   // 0..63
  const int lane = threadIdx.x & 31;
  uint32_t g = 0, pend_st = 0;
  bool pending = false;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int4 t = a.tiles[ti];
    const int N = (t.w + 15) & ~15;
    const __nv_bfloat16 *rows[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int n = tid + 64 * r;
      rows[r] = nullptr;
      if (n < N) {
        if (a.gather) {
          const int pos = a.off[t.x] + t.z + min(n, t.w - 1);
          rows[r] = a.bsrc + (size_t)a.ptok[pos] * a.ldb;
        } else {
          rows[r] = a.bsrc + (size_t)(a.poff[t.x] + t.z + n) * a.ldb;
        }
      }
    }
    bool ok = true;
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      const int st = g % PF_S;
      if (!pf_wait_warp(&b->empty[st], ((g / PF_S) & 1) ^ 1, b, a.status)) {
        ok = false;
        break;
      }
      uint8_t *B = sm + st * PF_STAGE + 2 * PF_A_BYTES;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (!rows[r]) continue;
        const int n = tid + 64 * r;
        const __nv_bfloat16 *src = rows[r] + s * PF_KS;
#pragma unroll
        for (int c = 0; c < 8; ++c) cp_async16(B + n * 128 + ((c ^ (n & 7)) << 4), src + c * 8);
      }
      cp_async_commit();
      if (pending) {
        cp_async_wait_1();
        tc05::fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b->b_full[pend_st]);
      }
      pending = true;
      pend_st = st;
    }
    if (!ok) break;
  }
  cp_async_wait_all();
  if (pending) {
    tc05::fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&b->b_full[pend_st]);
  }
}

__device__ void pf_mma(const PfGemm &a, uint8_t *sm, PfBars *b, int nt, uint32_t tmem) {
  const uint32_t base = smem_u32(sm);
  uint32_t g = 0, tc = 0;
  bool issued = false;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int4 t = a.tiles[ti];
    const uint32_t idesc = tc05::idesc_bf16_f32(PF_M, (t.w + 15) & ~15);
    if (!pf_wait(&b->acc_empty, (tc & 1) ^ 1, b, a.status)) goto done;
    tc05::fence_after_sync();
    for (int s = 0; s < a.ksteps; ++s, ++g) {
      const int st = g % PF_S;
      const uint32_t ph = (g / PF_S) & 1;
      if (!pf_wait(&b->a_full[st], ph, b, a.status) || !pf_wait(&b->b_full[st], ph, b, a.status)) goto done;
      tc05::fence_after_sync();
      issued = true;
      const uint32_t sa = base + st * PF_STAGE;
      const uint64_t d0 = tc05::sw128_desc(sa), d1 = tc05::sw128_desc(sa + PF_A_BYTES);
      const uint64_t db = tc05::sw128_desc(sa + 2 * PF_A_BYTES);
#pragma unroll
      for (int kk = 0; kk < PF_KS / 16; ++kk) {
        const uint32_t acc = (s | kk) != 0;
        tc05::mma_bf16(tmem, d0 + 2 * kk, db + 2 * kk, idesc, acc);
        tc05::mma_bf16(tmem + 256, d1 + 2 * kk, db + 2 * kk, idesc, acc);
      }
      tc05::commit(&b->empty[st]);
    }
    tc05::commit(&b->acc_full);
    ++tc;
  }
done:
  // every MMA this thread issued has completed before tensor memory is freed
  if (issued) {
    tc05::commit(&b->fin);
    if (!mbar_wait(&b->fin, 0, clock64() + WAIT_BUDGET_CYCLES)) set_status(a.status, DEV_TIMEOUT);
  }
}

__device__ __forceinline__ float silu(float v) { return v / (1.0f + __expf(-v)); }

__device__ void pf_epilogue(const PfGemm &a, PfBars *b, int nt, uint32_t tmem) {
  const int q = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
  const int r = 32 * q + lane;
  const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
  uint32_t tc = 0;
  for (int ti = blockIdx.x; ti < nt; ti += gridDim.x) {
    const int4 t = a.tiles[ti];
    const int N = (t.w + 15) & ~15;
    if (!pf_wait_warp(&b->acc_full, tc & 1, b, a.status)) return;
    tc05::fence_after_sync();
    if (a.mode == 0) {
      __nv_bfloat16 *h = a.hout + (size_t)(a.poff[t.x] + t.z) * a.ldh + t.y * PF_M + r;
      for (int c0 = 0; c0 < N; c0 += 16) {
        float gv[16], uv[16];
        tc05::ld16(tq + c0, gv);
        tc05::ld16(tq + 256 + c0, uv);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int n = c0 + i;
          const float hv = n < t.w ? silu(gv[i]) * uv[i] : 0.0f;
          h[(size_t)n * a.ldh] = __float2bfloat16_rn(hv);
        }
      }
    } else {
      const int pos0 = a.off[t.x] + t.z;
      float *yb = a.y + t.y * (2 * PF_M) + r;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        for (int c0 = 0; c0 < N; c0 += 16) {
          float v[16];
          tc05::ld16(tq + 256 * half + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = c0 + i;
            if (n < t.w) {
              const int pos = pos0 + n;
              atomicAdd(yb + half * PF_M + (size_t)a.ptok[pos] * a.ldy, a.pgate[pos] * v[i]);
            }
          }
        }
      }
    }
    tc05::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(&b->acc_empty);
    ++tc;
  }
}

__global__ void __launch_bounds__(PF_THREADS, 1) pf_gemm_kernel(const __grid_constant__ PfGemm a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  PfBars *b = reinterpret_cast<PfBars *>(sm + PF_OFF_BAR);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < PF_PS; ++i) {
      mbar_init(&b->pk_full[i], 1);
      mbar_init(&b->pk_empty[i], N_DEQ);
    }
    for (int i = 0; i < PF_S; ++i) {
      mbar_init(&b->a_full[i], N_DEQ);
      mbar_init(&b->b_full[i], N_BLOAD);
      mbar_init(&b->empty[i], 1);
    }
    mbar_init(&b->acc_full, 1);
    mbar_init(&b->acc_empty, 4);
    mbar_init(&b->fin, 1);
    b->abort = 0;
    fence_mbar_init();
  }
  if (warp == W_MMA) {
    tc05::tmem_alloc(&b->tmem_base, PF_TMEM_COLS);
    tc05::tmem_relinquish();
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = b->tmem_base;
  const int nt = *a.ntiles;

  if (warp == W_PRODUCER) {
    pf_producer(a, sm, b, nt);
  } else if (warp == W_MMA) {
    if ((threadIdx.x & 31) == 0) pf_mma(a, sm, b, nt, tmem);
    __syncwarp();
  } else if (warp < W_BLOAD + N_BLOAD) {
    pf_bload(a, sm, b, nt);
  } else if (warp < W_EPI + 4) {
    pf_epilogue(a, b, nt, tmem);
  } else {
    pf_dequant(a, sm, b, nt);
  }

  tc05::fence_before_sync();
  __syncthreads();
  if (warp == W_MMA) {
    tc05::fence_after_sync();
    tc05::tmem_dealloc(tmem, PF_TMEM_COLS);
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

// Tiles of at most 256 pairs per expert: the full 256-pair chunks first, in
// (expert, feature block, chunk) order, then each expert's remainder chunk,
// largest remainder first (ties by expert index), all feature blocks of one
// remainder adjacent. CTAs take tiles round-robin.
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
    for (int fb = 0; fb < a.fbs1; ++fb)
      for (int c = 0; c < nfull[r]; ++c)
        a.tiles1[(size_t)a.fbs1 * Fx + fb * nfull[r] + c] = make_int4(e, fb, c * PF_N, PF_N);
    for (int fb = 0; fb < a.fbs2; ++fb)
      for (int c = 0; c < nfull[r]; ++c)
        a.tiles2[(size_t)a.fbs2 * Fx + fb * nfull[r] + c] = make_int4(e, fb, c * PF_N, PF_N);
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
  size_t off, poff, perm, ptok, pgate, ntiles, tiles1, tiles2, h, total;
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
  L.tiles1 = o; o += up256(L.max_tiles1 * sizeof(int4));
  L.tiles2 = o; o += up256(L.max_tiles2 * sizeof(int4));
  L.h = o;      o += up256(L.h_rows * I * sizeof(__nv_bfloat16));
  L.total = o;
  return L;
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
                               qmoe_stream_t stream, void *const *events) {
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

  qmoe_status st = bucket_launch(idx, gate, T, k, E, off, perm, ptok, pgate, nullptr, nullptr, true, dev_status, s);
  if (st != QMOE_OK) return st;
  PlanArgs pa{off, E, I / PF_M, H / (2 * PF_M), poff, tiles1, tiles2, ntiles, dev_status};
  pf_plan_kernel<<<1, 1024, 0, s>>>(pa);
  note_launch();
  if (cudaGetLastError() != cudaSuccess) return QMOE_ERR_CUDA;
  if (cudaMemsetAsync(y, 0, (size_t)T * H * sizeof(float), s) != cudaSuccess) return QMOE_ERR_CUDA;

  const int bits = QMOE_Q4;
  PfGemm g1{};
  g1.w = static_cast<const uint8_t *>(ex->gate_up);
  g1.w_expert = expert_gu_bytes(bits, H, I);
  g1.tb = tile_bytes(bits, H);
  g1.cb = tile_code_bytes(bits, H);
  g1.fb_tiles = PF_M / 16;
  g1.a1_tiles = I / 16;
  g1.ksteps = H / PF_KS;
  g1.bsrc = static_cast<const __nv_bfloat16 *>(x);
  g1.ldb = H;
  g1.gather = 1;
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
  g2.w = static_cast<const uint8_t *>(ex->down);
  g2.w_expert = expert_dn_bytes(bits, H, I);
  g2.tb = tile_bytes(bits, I);
  g2.cb = tile_code_bytes(bits, I);
  g2.fb_tiles = 2 * PF_M / 16;
  g2.a1_tiles = PF_M / 16;
  g2.ksteps = I / PF_KS;
  g2.bsrc = h;
  g2.ldb = I;
  g2.gather = 0;
  g2.tiles = tiles2;
  g2.ntiles = ntiles + 1;
  g2.hout = nullptr;
  g2.y = y;
  g2.ldy = H;
  g2.mode = 1;
  st = pf_gemm_launch(g2, s);
  if (st != QMOE_OK) return st;
  if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[2]), s) != cudaSuccess) return QMOE_ERR_CUDA;
  return QMOE_OK;
}

extern "C" qmoe_status qmoe_ffn_prefill(const qmoe_experts *ex, const void *x, int T, const int32_t *idx,
                                        const float *gate, int k, float *y, void *workspace, size_t workspace_bytes,
                                        int32_t *dev_status, qmoe_stream_t stream) {
  return ffn_prefill(ex, x, T, idx, gate, k, y, workspace, workspace_bytes, dev_status, stream, nullptr);
}

extern "C" qmoe_status qmoe_ffn_prefill_timed(const qmoe_experts *ex, const void *x, int T, const int32_t *idx,
                                              const float *gate, int k, float *y, void *workspace,
                                              size_t workspace_bytes, int32_t *dev_status, qmoe_stream_t stream,
                                              void *const *events) {
  if (!events || !events[0] || !events[1] || !events[2]) return QMOE_ERR_INVALID_ARG;
  return ffn_prefill(ex, x, T, idx, gate, k, y, workspace, workspace_bytes, dev_status, stream, events);
}
