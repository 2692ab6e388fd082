// n-gram row gather ([P3] "Understanding the Architecture": a per-layer
// token-embedding table read a few rows at a time, 16 rows per token from a
// hash of its last three ids). Hash and row format are self-defined; the
// header states both. One warp per (token, slot): the token's hash and the
// slot's row, then the row's codes and block scales (160 bytes at D = 256)
// into registers and its D values out with streaming stores. Codes become
// floats by integer bit moves, not the conversion unit.
#include <cuda_fp16.h>

#include "common.cuh"

namespace qmoe {
namespace {

constexpr int NG_SLOTS = 16;
constexpr int NG_THREADS = 256;
constexpr int NG_WARPS = NG_THREADS / 32;
constexpr uint64_t NG_GAMMA = 0x9E3779B97F4A7C15ull;

// SplitMix64's output finaliser.
__device__ __forceinline__ uint64_t ng_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// A 4-bit code as a float without the conversion unit: 2^23 + q has q in its
// low mantissa bits, so subtracting 2^23 leaves q exactly.
__device__ __forceinline__ float code_f(uint32_t q) { return __fsub_rn(__uint_as_float(0x4B000000u | q), 8388608.0f); }

struct NgArgs {
  const int32_t *ngrams;   // [T][3]
  const uint8_t *codes;    // [R][D/2]
  const uint32_t *scales;  // [R][D/32]: fp16 d (low half), fp16 m (high half)
  float *out;              // [T][16][D]
  int32_t *rows;           // [T][16] or null
  uint64_t seed;
  long long R;
  int T, D;
};

__global__ void __launch_bounds__(NG_THREADS) ngram_gather_kernel(NgArgs a) {
  const int lane = threadIdx.x & 31;
  const long long nitems = (long long)a.T * NG_SLOTS;
  const int D = a.D;
  for (long long it = (long long)blockIdx.x * NG_WARPS + (threadIdx.x >> 5); it < nitems;
       it += (long long)gridDim.x * NG_WARPS) {
    const long long t = it / NG_SLOTS;
    const int i = (int)(it % NG_SLOTS);
    // every lane forms the same hash and row
    uint64_t h = ng_mix(a.seed + NG_GAMMA);
#pragma unroll
    for (int j = 0; j < 3; ++j) h = ng_mix(h ^ (uint64_t)(uint32_t)__ldg(a.ngrams + 3 * t + j));
    const uint64_t x = ng_mix(h + (uint64_t)(i + 1) * NG_GAMMA);
    const long long r = (long long)__umul64hi(x, (uint64_t)a.R);   // floor(x R / 2^64) < R
    if (lane == 0 && a.rows) a.rows[it] = (int32_t)r;
    const uint8_t *cr = a.codes + (size_t)r * (D / 2);
    const uint32_t *sr = a.scales + (size_t)r * (D / 32);
    float *o = a.out + (size_t)it * D;
    // lane l: elements 8l .. 8l + 7 of every 256-element chunk (one code word,
    // one block scale pair)
    for (int e0 = 8 * lane; e0 < D; e0 += 256) {
      const uint32_t cw = __ldg(reinterpret_cast<const uint32_t *>(cr + e0 / 2));
      const uint32_t dm = __ldg(sr + e0 / 32);
      const float d = __half2float(__ushort_as_half((unsigned short)(dm & 0xffffu)));
      const float m = __half2float(__ushort_as_half((unsigned short)(dm >> 16)));
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = __fmaf_rn(d, code_f((cw >> (4 * k)) & 15u), m);
      __stcs(reinterpret_cast<float4 *>(o + e0), make_float4(v[0], v[1], v[2], v[3]));
      __stcs(reinterpret_cast<float4 *>(o + e0 + 4), make_float4(v[4], v[5], v[6], v[7]));
    }
  }
}

}  // namespace
}  // namespace qmoe

using namespace qmoe;

extern "C" qmoe_status qmoe_ngram_gather(const int32_t *ngrams, int T, uint64_t seed, const uint8_t *codes,
                                         const uint16_t *scales, int64_t R, int D, float *out, int32_t *rows,
                                         qmoe_stream_t stream) {
  if (!ngrams || !codes || !scales || !out || T < 1 || R < 1) return QMOE_ERR_INVALID_ARG;
  if (R > 0x7fffffffLL) return QMOE_ERR_INVALID_ARG;
  if (D < 32 || D % 32 || D > 8192) return QMOE_ERR_UNSUPPORTED;
  const uintptr_t a4 = reinterpret_cast<uintptr_t>(ngrams) | reinterpret_cast<uintptr_t>(scales) |
                       reinterpret_cast<uintptr_t>(rows);
  if ((a4 & 3) || !aligned16(codes) || !aligned16(out)) return QMOE_ERR_INVALID_ARG;
  NgArgs a{ngrams, codes, reinterpret_cast<const uint32_t *>(scales), out, rows, seed, (long long)R, T, D};
  const long long want = ((long long)T * NG_SLOTS + NG_WARPS - 1) / NG_WARPS;
  const int grid = (int)(want < 16LL * num_sms() ? want : 16LL * num_sms());
  ngram_gather_kernel<<<grid, NG_THREADS, 0, (cudaStream_t)stream>>>(a);
  note_launch();
  return cuda_status(cudaGetLastError());
}
