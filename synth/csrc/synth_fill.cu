// Device side of the seeded synthetic generator: fills a layer's canonical
// code bytes and fp16 (d, m) pairs directly in GPU memory, bit-identical to
// synth/gen.py (checked by the GPU tests). Holds no arithmetic of the MoE
// method itself.
//
// SplitMix64 (Steele, Lea & Flood 2014) as a counter-based generator:
//   out(key, i) = mix64(key + (i + 1) * GAMMA)
// stream key of (seed, w0, w1, ...):
//   k = mix64(seed ^ KEY0); for each word w: k = mix64(k ^ ((w + 1) * GAMMA))
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t GAMMA = 0x9E3779B97F4A7C15ull;
constexpr uint64_t KEY0 = 0x6A09E667F3BCC909ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, int cfg, int layer, int expert, int what) {
  uint64_t k = mix64(seed ^ KEY0);
  k = mix64(k ^ ((uint64_t)(cfg + 1) * GAMMA));
  k = mix64(k ^ ((uint64_t)(layer + 1) * GAMMA));
  k = mix64(k ^ ((uint64_t)(expert + 1) * GAMMA));
  k = mix64(k ^ ((uint64_t)(what + 1) * GAMMA));
  return k;
}

// Codes: word i of expert e is out(key(seed, cfg, layer, e, what), i), stored
// little-endian; words_per_expert = code bytes per expert / 8.
__global__ void fill_codes(uint64_t seed, int cfg, int layer, int e0, int E, int what, size_t words_per_expert,
                           uint64_t *dst) {
  size_t total = (size_t)E * words_per_expert;
  for (size_t w = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w < total; w += (size_t)gridDim.x * blockDim.x) {
    int e = (int)(w / words_per_expert);
    size_t i = w % words_per_expert;
    uint64_t key = stream_key(seed, cfg, layer, e0 + e, what);
    dst[w] = mix64(key + (uint64_t)(i + 1) * GAMMA);
  }
}

// Scales: block j of expert e: u = (out(key, j) >> 11) * 2^-53,
// d = fp16_rne(lo + span * u) (no fused multiply-add), m = fp16_rne(-c * d).
__global__ void fill_scales(uint64_t seed, int cfg, int layer, int e0, int E, int what, size_t blocks_per_expert,
                            double lo, double span, double c, uint32_t *dst) {
  size_t total = (size_t)E * blocks_per_expert;
  for (size_t j = blockIdx.x * (size_t)blockDim.x + threadIdx.x; j < total; j += (size_t)gridDim.x * blockDim.x) {
    int e = (int)(j / blocks_per_expert);
    size_t b = j % blocks_per_expert;
    uint64_t key = stream_key(seed, cfg, layer, e0 + e, what);
    uint64_t r = mix64(key + (uint64_t)(b + 1) * GAMMA);
    double u = __dmul_rn((double)(r >> 11), 1.1102230246251565e-16);  // 2^-53, exact
    double d = __dadd_rn(lo, __dmul_rn(span, u));
    __half d16 = __double2half(d);
    double m = __dmul_rn(-c, (double)__half2float(d16));
    __half m16 = __double2half(m);
    dst[j] = (uint32_t)__half_as_ushort(d16) | ((uint32_t)__half_as_ushort(m16) << 16);
  }
}

int grid_for(size_t n) {
  size_t b = (n + 255) / 256;
  return (int)(b > 148 * 32 ? 148 * 32 : (b ? b : 1));
}

}  // namespace

extern "C" int synth_fill_codes(uint64_t seed, int cfg, int layer, int e0, int E, int what, size_t bytes_per_expert,
                                void *dst, void *stream) {
  if (!dst || E <= 0 || bytes_per_expert % 8) return 1;
  size_t wpe = bytes_per_expert / 8;
  fill_codes<<<grid_for((size_t)E * wpe), 256, 0, (cudaStream_t)stream>>>(seed, cfg, layer, e0, E, what, wpe,
                                                                          static_cast<uint64_t *>(dst));
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" int synth_fill_scales(uint64_t seed, int cfg, int layer, int e0, int E, int what, size_t blocks_per_expert,
                                 double lo, double span, double c, void *dst, void *stream) {
  if (!dst || E <= 0) return 1;
  fill_scales<<<grid_for((size_t)E * blocks_per_expert), 256, 0, (cudaStream_t)stream>>>(
      seed, cfg, layer, e0, E, what, blocks_per_expert, lo, span, c, static_cast<uint32_t *>(dst));
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
