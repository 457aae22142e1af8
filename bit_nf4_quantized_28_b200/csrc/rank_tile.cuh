// rank_tile.cuh -- one 64 x 128 tile of a rank-r product P = L R, L [rows, r]
// and R [r, cols] in bf16, accumulated in fp32 on the tensor cores
// (mma.sync m16n8k16) by a CTA of 128 threads, for kernels that add P to an
// HBM-bound elementwise result (the LoRA merge, the dropout dx update).
//
//  1. L rows n0..n0+63 and R columns k0..k0+127 are copied to shared memory,
//     zero padded to a multiple of 16 in r, past the last row and past the
//     last column;
//  2. each warp computes 16 rows x 128 columns (R read with ldmatrix .trans)
//     into registers (rank_tile_mma), or into the fp32 tile ps [64][kTilePPad]
//     in shared memory (rank_tile_product).
#pragma once

#include "common.cuh"
#include "lora_small.cuh"

namespace qn {

constexpr int kTileRows = 64;
constexpr int kTileCols = 128;
constexpr int kTileThreads = 128;
constexpr int kTileRPad = kTileCols + 8;     // bf16 per row of the staged R columns
constexpr int kTilePPad = kTileCols + 4;     // floats per row of the product tile

__host__ __device__ constexpr int rank_tile_r16(int r) { return (r + 15) & ~15; }

// Shared memory of the staged operands for rank r: L rows [64][r16 + 8] and
// R columns [r16][kTileRPad].
__host__ __device__ constexpr size_t rank_tile_operand_bytes(int r) {
  return r > 0 ? static_cast<size_t>(kTileRows) * (rank_tile_r16(r) + 8) * 2 +
                     static_cast<size_t>(rank_tile_r16(r)) * kTileRPad * 2
               : 0;
}

// Stages L rows n0..n0+63 and R columns k0..k0+127 in shared memory and
// computes warp w's rows 16w..16w+15 of the tile into acc in the m16n8k16
// accumulator layout: acc[t] holds (row 16w + g, columns 8t + 2q, +1) in
// [0], [1] and (row 16w + g + 8, the same columns) in [2], [3], where
// g = lane / 4 and q = lane % 4.  L is [nrows, r] row-major, R is [r, K]
// row-major; r is a multiple of 8.  ops points at rank_tile_operand_bytes(r)
// bytes of 16-byte aligned shared memory.
__device__ __forceinline__ void rank_tile_mma(const __nv_bfloat16* L, int64_t nrows, const __nv_bfloat16* R,
                                              int64_t K, int r, int64_t n0, int64_t k0, __nv_bfloat16* ops,
                                              float (&acc)[16][4]) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r16 = rank_tile_r16(r);
  const int lpad = r16 + 8;
  __nv_bfloat16* ls = ops;                        // [64][lpad]
  __nv_bfloat16* rs = ops + kTileRows * lpad;     // [r16][kTileRPad]
  // L rows, columns 0..r16-1 (zero past r and past the last row), 8 bf16 per copy
  for (int i = tid; i < kTileRows * (r16 / 8); i += kTileThreads) {
    const int row = i / (r16 / 8), c8 = (i % (r16 / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (c8 < r && n0 + row < nrows) v = *reinterpret_cast<const uint4*>(L + (n0 + row) * r + c8);
    *reinterpret_cast<uint4*>(ls + row * lpad + c8) = v;
  }
  // R rows 0..r16-1 (zero past r), columns k0..k0+127 (zero past K)
  for (int i = tid; i < r16 * (kTileCols / 8); i += kTileThreads) {
    const int j = i / (kTileCols / 8), c8 = (i % (kTileCols / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (j < r && k0 + c8 < K) v = *reinterpret_cast<const uint4*>(R + static_cast<int64_t>(j) * K + k0 + c8);
    *reinterpret_cast<uint4*>(rs + j * kTileRPad + c8) = v;
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  const int mi = lane >> 3, rr = lane & 7;
  for (int kk = 0; kk < r16; kk += 16) {
    uint32_t a0, a1, a2, a3;
    // A operand L[m][j]: (m 0-7, j 0-7), (m 8-15, j 0-7), (m 0-7, j 8-15), (m 8-15, j 8-15)
    ldsm_x4(smem_u32(ls + (warp * 16 + (mi & 1) * 8 + rr) * lpad + kk + (mi >> 1) * 8), a0, a1, a2, a3);
#pragma unroll
    for (int t = 0; t < 16; t += 2) {
      uint32_t b0, b1, b2, b3;
      // B operand R[j][col], j-major in shared memory, read transposed:
      // (j 0-7, col 0-7), (j 8-15, col 0-7), (j 0-7, col 8-15), (j 8-15, col 8-15)
      ldsm_x4_t(smem_u32(rs + (kk + (mi & 1) * 8 + rr) * kTileRPad + 8 * t + (mi >> 1) * 8), b0, b1, b2, b3);
      mma_bf16_16816(acc[t], a0, a1, a2, a3, b0, b1);
      mma_bf16_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
    }
  }
}

// P[n0 .. n0+63][k0 .. k0+127] -> ps [64][kTilePPad] (fp32), each warp its
// own 16 rows; the caller synchronizes before reading other warps' rows.
__device__ __forceinline__ void rank_tile_product(const __nv_bfloat16* L, int64_t nrows,
                                                  const __nv_bfloat16* R, int64_t K, int r, int64_t n0,
                                                  int64_t k0, float* ps, __nv_bfloat16* ops) {
  float acc[16][4];
  rank_tile_mma(L, nrows, R, K, r, n0, k0, ops, acc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    const int col = 8 * t + 2 * q, row = warp * 16 + g;
    *reinterpret_cast<float2*>(ps + row * kTilePPad + col) = make_float2(acc[t][0], acc[t][1]);
    *reinterpret_cast<float2*>(ps + (row + 8) * kTilePPad + col) = make_float2(acc[t][2], acc[t][3]);
  }
}

}  // namespace qn
