// mma_tiles.cuh -- 16-row tile products on the warp-level tensor-core path
// (m16n8k16, bf16 in, fp32 accumulate) over [rows][64] bf16 tiles stored in
// shared memory with the 128-byte TMA swizzle (ptx::sw128).
//
// Fragment conventions (one warp, lane = 4 * gq + tq4):
//   * a C tile c[j][e] (16 x 16, fp32) holds rows gq (e = 0, 1) and gq + 8
//     (e = 2, 3), columns 8 j + 2 tq4 + (e & 1);
//   * an A fragment a[4] (16 x 16, bf16 pairs) holds the same elements in the
//     order {rows 0-7 cols 0-7, rows 8-15 cols 0-7, rows 0-7 cols 8-15,
//     rows 8-15 cols 8-15}, which is what pack_a() builds from a C tile.
#pragma once

#include "ptx.cuh"

namespace llsa {
namespace tiles {

// A fragments of a 16 x 64 tile (rows = M, columns = the contracted d), four
// k-steps of 16 columns; the tile's rows start at `row0`.
__device__ __forceinline__ void load_a(uint32_t (*a)[4], uint32_t tile, int lane, int row0 = 0) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const int row = row0 + (lane & 15);
    const int col = ks * 16 + ((lane >> 4) << 3);
    ptx::ldmatrix_x4(tile + ptx::sw128(row, col), a[ks][0], a[ks][1], a[ks][2], a[ks][3]);
  }
}

// C (16 x 16) = A (16 x 64, fragments) * T^T, where T is rows row0..row0+15 of
// a [rows][64] tile: each output column is one row of T.
__device__ __forceinline__ void mma_abt(float (*c)[4], const uint32_t (*a)[4], uint32_t tile, int row0, int lane) {
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) c[j][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const int row = row0 + (lane & 7) + ((lane >> 4) << 3);
    const int col = ks * 16 + (((lane >> 3) & 1) << 3);
    uint32_t b0, b1, b2, b3;
    ptx::ldmatrix_x4(tile + ptx::sw128(row, col), b0, b1, b2, b3);
    ptx::mma_bf16(c[0], a[ks], b0, b1);
    ptx::mma_bf16(c[1], a[ks], b2, b3);
  }
}

// acc (16 x 64) += A (16 x 16, one fragment) * T, where T is rows
// row0..row0+15 of a [rows][64] tile (the contracted index runs over T's rows).
__device__ __forceinline__ void mma_ab(float (*acc)[4], const uint32_t* a, uint32_t tile, int row0, int lane) {
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    const int row = row0 + (lane & 7) + (((lane >> 3) & 1) << 3);
    const int col = (j + (lane >> 4)) * 8;
    uint32_t b0, b1, b2, b3;
    ptx::ldmatrix_x4_trans(tile + ptx::sw128(row, col), b0, b1, b2, b3);
    ptx::mma_bf16(acc[j], a, b0, b1);
    ptx::mma_bf16(acc[j + 1], a, b2, b3);
  }
}

// A fragment (bf16) of a C tile.
__device__ __forceinline__ void pack_a(uint32_t* a, const float (*c)[4]) {
  a[0] = ptx::pack_bf16(c[0][0], c[0][1]);
  a[1] = ptx::pack_bf16(c[0][2], c[0][3]);
  a[2] = ptx::pack_bf16(c[1][0], c[1][1]);
  a[3] = ptx::pack_bf16(c[1][2], c[1][3]);
}

// A fragment of the transpose of the 16 x 16 matrix whose fragment is `a`.
__device__ __forceinline__ void transpose_a(uint32_t* t, const uint32_t* a) {
  t[0] = ptx::movmatrix_trans(a[0]);
  t[1] = ptx::movmatrix_trans(a[2]);
  t[2] = ptx::movmatrix_trans(a[1]);
  t[3] = ptx::movmatrix_trans(a[3]);
}

__device__ __forceinline__ void zero_acc(float (*acc)[4]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
}

// Sums over the 4 lanes of a quad (one C-tile row) and over the 8 quads
// (one C-tile column).
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}
__device__ __forceinline__ float column_sum8(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  return v + __shfl_xor_sync(0xffffffffu, v, 16);
}

}  // namespace tiles
}  // namespace llsa
