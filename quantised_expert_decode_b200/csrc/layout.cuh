// Packed device layout of the block-quantised expert matrices.
//
// A matrix [rows, K] (K = reduction axis) is stored as 16-row tiles. A tile
// holds the codes of its 16 rows x K, then one 32-bit (d | m << 16) word per
// (block, row):
//
//   codes : Q2 groups of 4 blocks, Q4 groups of 2 blocks; a group is 512 bytes
//           = 32 lanes x 16 bytes, so lane l of a warp reads one uint4 holding
//           its integer-MMA A fragments for every block of the group.
//   scales: [K/32 blocks][8 groups g][2 (row g, row g+8)] x u32.
//
// Within a block, lane (g = l/4, t = l%4) owns the 16 codes of fragment
// registers r = 0..3 (m16n8k32 A layout):
//   r=0: row g,   k = 4t+i      r=1: row g+8, k = 4t+i
//   r=2: row g,   k = 16+4t+i   r=3: row g+8, k = 16+4t+i      (i = 0..3)
// Q2: one u32 per block, code (r, i) at bits 8i + 2r, so register r is
//     (w >> 2r) & 0x03030303.
// Q4: two u32 per block, word r/2 holds code (r, i) at bits 8i + 4(r%2), so
//     register r is (w[r/2] >> 4(r%2)) & 0x0F0F0F0F.
#pragma once

#include <stdint.h>

namespace qmoe {

__host__ __device__ constexpr int tile_code_bytes(int bits, int K) { return 2 * K * bits; }
__host__ __device__ constexpr int tile_scale_bytes(int K) { return 2 * K; }
__host__ __device__ constexpr int tile_bytes(int bits, int K) { return 2 * K * (bits + 1); }
__host__ __device__ constexpr int blocks_per_group(int bits) { return bits == 2 ? 4 : 2; }

// Packed bytes of all gate+up tiles of one expert and of its down tiles.
__host__ __device__ constexpr size_t expert_gu_bytes(int bits, int H, int I) {
  return (size_t)2 * (I / 16) * tile_bytes(bits, H);
}
__host__ __device__ constexpr size_t expert_dn_bytes(int bits, int H, int I) {
  return (size_t)(H / 16) * tile_bytes(bits, I);
}

// (row offset inside the tile, k offset inside the block) of fragment register r, element i
__host__ __device__ inline void frag_pos(int lane, int r, int i, int &row, int &kk) {
  int g = lane >> 2, t = lane & 3;
  row = g + ((r & 1) ? 8 : 0);
  kk = ((r & 2) ? 16 : 0) + 4 * t + i;
}

}  // namespace qmoe
