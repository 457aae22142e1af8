// merge.cuh -- the LoRA adapter folded into the dequantized weight.
//
// [LoRA y QLoRA en Profundidad, "Cómo Funciona LoRA": for inference the LoRA
//  matrices are merged, W_final = W + (alpha / r) B @ A.  QLoRA glossary,
//  "Compromessi": merging into the 4-bit base model first dequantizes it to
//  16 bits.]
//
//   W_out[n][k] = bf16( fl32(W_hat[n][k]) + fl32(s * sum_j B[n][j] A[j][k]) ),
//   W_hat = bf16(fl32(level[code] * s_hat))   (the same W_hat as dequantize)
//
// HBM-bound: codes (0.5 B per weight) in, bf16 (2 B per weight) out; A and B
// are re-read from L2.  A CTA owns a tile of 64 rows x 128 columns:
//  1. P = B A for the tile is computed on the tensor cores into shared
//     memory (rank_tile_product);
//  2. each thread then takes 8 consecutive weights of a row (its code word
//     and scale parts were loaded at the start): the staged P values, one
//     16-byte store.
#pragma once

#include "common.cuh"
#include "nf4_storage.cuh"
#include "rank_tile.cuh"

namespace qn {

constexpr int kMergeRows = kTileRows;
constexpr int kMergeCols = kTileCols;
constexpr int kMergeThreads = kTileThreads;
constexpr int kMergeItems = kMergeRows * (kMergeCols / 8) / kMergeThreads;   // 8-weight items per thread

// Shared memory for rank r: levels, the product tile and the staged B rows
// and A columns; sized per launch, so that a small rank leaves room for more
// CTAs per SM.
__host__ __device__ constexpr size_t merge_smem_bytes(int r) {
  return 16 * 4 + static_cast<size_t>(kMergeRows) * kTilePPad * 4 + rank_tile_operand_bytes(r);
}

struct MergeParams {
  const uint8_t* codes;       // [N, K/2]
  const int8_t* qscale;       // [N*K/64]
  const float* dq_step;
  const float* dq_mean;
  const __nv_bfloat16* A;     // [r, K] (r > 0)
  const __nv_bfloat16* B;     // [N, r] (r > 0)
  __nv_bfloat16* out;         // [N, K]
  int64_t N, K;
  int r;                      // 0 or a multiple of 8, <= kMaxRank
  float s;                    // fl32(alpha / r)
  Levels lv;
};

__global__ void __launch_bounds__(kMergeThreads) qlora_merge_kernel(MergeParams p) {
  extern __shared__ __align__(16) uint8_t merge_smem[];
  const int r = p.r;
  float* lv = reinterpret_cast<float*>(merge_smem);                                           // [16]
  float* ps = lv + 16;                                                                        // [64][PPad]
  __nv_bfloat16* ops = reinterpret_cast<__nv_bfloat16*>(ps + kMergeRows * kTilePPad);         // operands

  pdl_launch_dependents();
  pdl_wait_primary();
  const int tid = threadIdx.x;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kMergeRows;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kMergeCols;
  if (tid < 16) lv[tid] = p.lv.v[tid];

  // this thread's 8-weight items: code words and raw scale parts, loaded
  // first so that their latency overlaps the product below
  const int64_t half_k = p.K >> 1, kb = p.K >> 6;
  uint32_t cw[kMergeItems];
  int8_t sq[kMergeItems];
  float sst[kMergeItems], smn[kMergeItems];
#pragma unroll
  for (int it = 0; it < kMergeItems; ++it) {
    const int i = tid + it * kMergeThreads;
    const int row = i / (kMergeCols / 8), c8 = (i % (kMergeCols / 8)) * 8;
    const int64_t n = n0 + row, k = k0 + c8;
    cw[it] = 0; sq[it] = 0; sst[it] = 0.f; smn[it] = 0.f;
    if (k < p.K) {
      cw[it] = *reinterpret_cast<const uint32_t*>(p.codes + n * half_k + (k >> 1));
      const int64_t blk = n * kb + (k >> 6);
      sq[it] = p.qscale[blk];
      sst[it] = p.dq_step[blk >> 8];
      smn[it] = p.dq_mean[blk >> 8];
    }
  }

  if (r > 0) rank_tile_product(p.B, p.N, p.A, p.K, r, n0, k0, ps, ops);
  __syncthreads();

  // 8 consecutive weights per item: 64 rows x 16 items
  const float s = p.s;
#pragma unroll
  for (int it = 0; it < kMergeItems; ++it) {
    const int i = tid + it * kMergeThreads;
    const int row = i / (kMergeCols / 8), c8 = (i % (kMergeCols / 8)) * 8;
    const int64_t n = n0 + row, k = k0 + c8;
    if (k >= p.K) continue;
    const float sh = restore_scale(sq[it], sst[it], smn[it]);
    float extra[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) extra[e] = 0.f;
    if (r > 0) {
      const float4 p0 = *reinterpret_cast<const float4*>(ps + row * kTilePPad + c8);
      const float4 p1 = *reinterpret_cast<const float4*>(ps + row * kTilePPad + c8 + 4);
      const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) extra[e] = __fmul_rn(s, pv[e]);
    }
    uint32_t packed[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      // element 2j of a row sits in the low nibble of byte j
      const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[(cw[it] >> (4 * e)) & 15u], sh)));
      const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[(cw[it] >> (4 * e + 4)) & 15u], sh)));
      packed[e / 2] = pack_bf16x2(__fadd_rn(w0, extra[e]), __fadd_rn(w1, extra[e + 1]));
    }
    *reinterpret_cast<uint4*>(p.out + n * p.K + k) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
}

}  // namespace qn
