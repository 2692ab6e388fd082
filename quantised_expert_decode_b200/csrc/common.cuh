// Device helpers shared by libqmoe's kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "qmoe.h"

namespace qmoe {

// ------------------------------------------------------------------ host --
void note_launch(int n = 1);
qmoe_status cuda_status(cudaError_t e);
int num_sms();
size_t max_smem_optin();

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// device status codes written to *dev_status (first error wins)
constexpr int32_t DEV_OK = 0;
constexpr int32_t DEV_BAD_INDEX = 1;
constexpr int32_t DEV_DUP_INDEX = 2;
constexpr int32_t DEV_TIMEOUT = 3;
constexpr int32_t DEV_RANGE = 4;   // a decode partial sum too large for the exact fixed-point sums

// Time budget of every device-side wait, in SM clock cycles (~1 s at 2 GHz).
constexpr long long WAIT_BUDGET_CYCLES = 2000000000LL;

__device__ __forceinline__ void set_status(int32_t *st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

// ------------------------------------------------------------ smem / PTX --
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase. Returns false when the budget ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long deadline) {
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() > deadline) return false;
  }
  return true;
}

// Bulk asynchronous copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 policy for bytes read once per pass (expert and router weights): evicted
// first, so that the streamed weights do not push the kernels' code, the
// activations and the small shared buffers out of L2.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// bulk_g2s with an L2 cache policy (l2_evict_first for streamed weights).
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Integer tensor-core MMA: D[16x8] += A[16x32] (u8 codes) * B[32x8] (s8 limbs).
// Fragments per lane (g = lane/4, t = lane%4):
//   a0: A[g][4t..4t+3]   a1: A[g+8][4t..4t+3]   a2: A[g][16+4t..]   a3: A[g+8][16+4t..]
//   b0: B[4t..4t+3][g]   b1: B[16+4t..16+4t+3][g]
//   d0,d1: D[g][2t], D[g][2t+1]   d2,d3: D[g+8][2t], D[g+8][2t+1]
__device__ __forceinline__ void mma_u8s8(int &d0, int &d1, int &d2, int &d3, uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d0), "+r"(d1), "+r"(d2), "+r"(d3)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Orders this thread's generic-proxy memory accesses (and those it has
// synchronised with) before its subsequent async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async;" ::: "memory"); }

// Programmatic dependent launch: wait for the preceding grid's completion (and
// its memory) / allow the next grid on the stream to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Grid-wide barrier for a co-resident grid (cooperative launch). Called by one
// thread per CTA after its CTA-local barrier; the caller fences after it. The
// counter's top bit flips once per barrier: CTA 0 adds 0x80000000 - (G-1),
// every other CTA adds 1, so the total added per barrier is exactly
// 0x80000000, the low bits return to 0 and the flip comes with the last
// arrival, whatever the order. A fence publishes this CTA's writes (ordered
// before it by the CTA barrier), then a relaxed atomic add arrives; the last
// arrival sees the flip in the value its own add returns, the others poll with
// plain loads. The caller's fence after the barrier makes everyone else's
// writes visible (measured: relaxed add and plain polling cost 0.2 us less
// per barrier than an acquire-release add and acquire loads). Returns false
// when the wait ran out of its budget.
__device__ __forceinline__ bool grid_barrier_one_thread(unsigned *bar, unsigned nblocks) {
  const unsigned inc = (blockIdx.x == 0) ? (0x80000000u - (nblocks - 1u)) : 1u;
  __threadfence();   // cumulative: covers the writes of the CTA ordered before by its barrier
  const unsigned old = atomicAdd(bar, inc);
  if (((old + inc) ^ old) & 0x80000000u) return true;
  const long long deadline = clock64() + WAIT_BUDGET_CYCLES;
  while (((*reinterpret_cast<volatile unsigned *>(bar) ^ old) & 0x80000000u) == 0u) {
    if (clock64() > deadline) return false;
  }
  return true;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive warp scan of three counters at once.
__device__ __forceinline__ void warp_scan3(int &a, int &b, int &c) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, a, o);
    const int y = __shfl_up_sync(0xffffffffu, b, o);
    const int z = __shfl_up_sync(0xffffffffu, c, o);
    if (lane >= o) {
      a += x;
      b += y;
      c += z;
    }
  }
}

// Orderable unsigned key of a float (larger float -> larger key; every key > 0
// for non-NaN input; 0 marks "no value").
__device__ __forceinline__ unsigned float_key(float f) {
  unsigned b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

}  // namespace qmoe
