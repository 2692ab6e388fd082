// qmoe_pack: canonical block-format bytes -> packed tensor-core tile layout.
#include "common.cuh"
#include "layout.cuh"

namespace qmoe {
namespace {

struct PackArgs {
  const uint8_t *codes[2];
  const uint16_t *scales[2];
  uint32_t *dst;
  int bits, nmat, E, rows, K;
};

__device__ __forceinline__ uint32_t canon_code(const uint8_t *codes, int bits, int K, int row, int k) {
  int per = 8 / bits;
  uint32_t byte = codes[(size_t)row * (K / per) + k / per];
  return (byte >> (bits * (k % per))) & ((1u << bits) - 1u);
}

// One thread per 32-bit word of the packed output.
__global__ void pack_kernel(PackArgs a) {
  const int K = a.K, bits = a.bits;
  const int tiles = a.rows / 16;
  const int cw = tile_code_bytes(bits, K) / 4;   // code words per tile
  const int sw = tile_scale_bytes(K) / 4;        // scale words per tile
  const int tw = cw + sw;
  const size_t total = (size_t)a.E * a.nmat * tiles * tw;
  for (size_t w = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w < total; w += (size_t)gridDim.x * blockDim.x) {
    size_t tile_id = w / tw;
    int in = (int)(w % tw);
    int tile = (int)(tile_id % tiles);
    size_t em = tile_id / tiles;
    int mat = (int)(em % a.nmat);
    size_t e = em / a.nmat;
    const uint8_t *codes = a.codes[mat] + e * (size_t)a.rows * (K * bits / 8);
    const uint16_t *scales = a.scales[mat] + e * (size_t)a.rows * (K / 32) * 2;
    uint32_t out = 0;
    if (in < cw) {
      int group = in / 128, rem = in % 128, lane = rem / 4;
      int blk, r0, nreg;
      if (bits == 2) {
        blk = group * 4 + (rem % 4);
        r0 = 0;
        nreg = 4;
      } else {
        blk = group * 2 + (rem % 4) / 2;
        r0 = 2 * (rem % 2);
        nreg = 2;
      }
      for (int rr = 0; rr < nreg; ++rr) {
        int r = r0 + rr;
        for (int i = 0; i < 4; ++i) {
          int row, kk;
          frag_pos(lane, r, i, row, kk);
          uint32_t q = canon_code(codes, bits, K, tile * 16 + row, blk * 32 + kk);
          int shift = (bits == 2) ? (8 * i + 2 * r) : (8 * i + 4 * rr);
          out |= q << shift;
        }
      }
    } else {
      int s = in - cw;               // [blk][g][j]
      int blk = s / 16, g = (s % 16) / 2, j = s % 2;
      int row = tile * 16 + g + 8 * j;
      const uint16_t *p = scales + ((size_t)row * (K / 32) + blk) * 2;
      out = (uint32_t)p[0] | ((uint32_t)p[1] << 16);
    }
    a.dst[w] = out;
  }
}

}  // namespace
}  // namespace qmoe

using namespace qmoe;

extern "C" size_t qmoe_packed_bytes(int fmt, int kind, int E, int H, int I) {
  if ((fmt != QMOE_Q2 && fmt != QMOE_Q4) || E <= 0 || H <= 0 || I <= 0) return 0;
  if (kind == QMOE_GATE_UP) return (size_t)E * expert_gu_bytes(fmt, H, I);
  if (kind == QMOE_DOWN) return (size_t)E * expert_dn_bytes(fmt, H, I);
  return 0;
}

extern "C" qmoe_status qmoe_pack(int fmt, int kind, int E, int H, int I, const uint8_t *codes_a,
                                 const uint16_t *scales_a, const uint8_t *codes_up, const uint16_t *scales_up,
                                 void *dst, size_t dst_bytes, qmoe_stream_t stream) {
  if (fmt != QMOE_Q2 && fmt != QMOE_Q4) return QMOE_ERR_UNSUPPORTED;
  if (kind != QMOE_GATE_UP && kind != QMOE_DOWN) return QMOE_ERR_INVALID_ARG;
  if (E <= 0 || H <= 0 || I <= 0) return QMOE_ERR_INVALID_ARG;
  if (H % 128 || I % 128) return QMOE_ERR_UNSUPPORTED;
  if (!codes_a || !scales_a || !dst) return QMOE_ERR_INVALID_ARG;
  if (kind == QMOE_GATE_UP && (!codes_up || !scales_up)) return QMOE_ERR_INVALID_ARG;
  if (!aligned16(dst)) return QMOE_ERR_INVALID_ARG;
  size_t need = qmoe_packed_bytes(fmt, kind, E, H, I);
  if (dst_bytes < need) return QMOE_ERR_INVALID_ARG;
  PackArgs a;
  a.bits = fmt;
  a.E = E;
  a.dst = static_cast<uint32_t *>(dst);
  if (kind == QMOE_GATE_UP) {
    a.nmat = 2;
    a.rows = I;
    a.K = H;
    a.codes[0] = codes_a;
    a.codes[1] = codes_up;
    a.scales[0] = scales_a;
    a.scales[1] = scales_up;
  } else {
    a.nmat = 1;
    a.rows = H;
    a.K = I;
    a.codes[0] = a.codes[1] = codes_a;
    a.scales[0] = a.scales[1] = scales_a;
  }
  size_t words = need / 4;
  int blocks = (int)((words + 255) / 256);
  if (blocks > 148 * 64) blocks = 148 * 64;
  pack_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(a);
  note_launch();
  return cuda_status(cudaGetLastError());
}
