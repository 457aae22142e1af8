// dropout.cuh -- LoRA dropout: the keep mask, the masked LoRA input, and the
// masked LoRA term of dx.
//
// [LoRA y QLoRA en Profundidad, "Dropout (lora_dropout)": during training
//  the dropout of the LoRA layers zeroes randomly chosen elements, as
//  regularisation; 0.05 in the lesson's config.]
//
// With keep the mask and p the rate, the layer computes
//     y  = x W_hat^T + s_d (x_m A^T) B^T,   x_m = x * keep,  s_d = s / (1 - p)
//     dx = dy W_hat + s_d keep * ((dy B) A)
//     dA = s_d (dy B)^T x_m,   dB = s_d dy^T (x_m A^T)
// which is the inverted dropout x * keep / (1 - p) on the LoRA path with its
// 1 / (1 - p) moved into the scale: x_m is exact in bf16, and the rank-r
// kernels read it as they read x.
//
// The draw is Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011): element e of x (row-major) takes
// word e % 4 of the block for counter (e / 4 as two words, offset as two
// words) under key = seed, and is kept iff the word >= floor(p * 2^32).
// The keep mask is one bit per element, bit e % 32 of 32-bit word e / 32.
#pragma once

#include "common.cuh"
#include "rank_tile.cuh"

namespace qn {

// One Philox4x32 block of ten rounds.  Each round takes the double-width
// products of words 0 and 2 with the round multipliers; the key advances by
// the Weyl increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    if (i > 0) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint64_t p0 = static_cast<uint64_t>(kM0) * c.x;   // one 32 x 32 -> 64-bit multiply
    const uint64_t p1 = static_cast<uint64_t>(kM1) * c.z;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k0, static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k1, static_cast<uint32_t>(p0));
  }
  return c;
}

// Keep bits of elements 8i .. 8i+7 (bit b for element 8i + b): Philox
// blocks 2i and 2i + 1.
__device__ __forceinline__ uint32_t keep_bits8(uint64_t i, uint32_t key0, uint32_t key1, uint32_t off0,
                                               uint32_t off1, uint32_t thresh) {
  const uint64_t q = 2 * i;
  const uint4 a = philox4x32_10(make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32), off0, off1),
                                key0, key1);
  const uint4 b = philox4x32_10(
      make_uint4(static_cast<uint32_t>(q + 1), static_cast<uint32_t>((q + 1) >> 32), off0, off1), key0, key1);
  return static_cast<uint32_t>(a.x >= thresh) | (static_cast<uint32_t>(a.y >= thresh) << 1) |
         (static_cast<uint32_t>(a.z >= thresh) << 2) | (static_cast<uint32_t>(a.w >= thresh) << 3) |
         (static_cast<uint32_t>(b.x >= thresh) << 4) | (static_cast<uint32_t>(b.y >= thresh) << 5) |
         (static_cast<uint32_t>(b.z >= thresh) << 6) | (static_cast<uint32_t>(b.w >= thresh) << 7);
}

struct DropoutParams {
  const uint4* x;        // [n8] groups of 8 bf16
  uint4* xm;             // [n8] x * keep
  uint32_t* keep;        // [n8 / 4]
  int64_t n8;            // elements / 8, a multiple of 4
  uint32_t key0, key1;   // seed
  uint32_t off0, off1;   // offset
  uint32_t thresh;       // floor(p * 2^32)
};

constexpr int kDropoutThreads = 256;

// Each warp takes chunks of 128 groups of 8 elements (2 KB of x): lane l
// handles groups 32 j + l of the chunk, so every load and store of a warp
// is 512 contiguous bytes; four lanes' 8-bit masks make one keep word.
__global__ void __launch_bounds__(kDropoutThreads) lora_dropout_kernel(DropoutParams p) {
  pdl_launch_dependents();
  pdl_wait_primary();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kDropoutThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kDropoutThreads) >> 5;
  const int64_t chunks = (p.n8 + 127) / 128;
  for (int64_t c = warp; c < chunks; c += nwarps) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = c * 128 + 32 * j + lane;
      v[j] = i < p.n8 ? p.x[i] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = c * 128 + 32 * j + lane;
      const bool ok = i < p.n8;
      const uint32_t bits = ok ? keep_bits8(static_cast<uint64_t>(i), p.key0, p.key1, p.off0, p.off1, p.thresh) : 0u;
      // bf16 element 2w of the group is the low half of 32-bit word w
      uint32_t m[4];
#pragma unroll
      for (int w = 0; w < 4; ++w)
        m[w] = (((bits >> (2 * w)) & 1u) ? 0x0000FFFFu : 0u) | (((bits >> (2 * w + 1)) & 1u) ? 0xFFFF0000u : 0u);
      if (ok) p.xm[i] = make_uint4(v[j].x & m[0], v[j].y & m[1], v[j].z & m[2], v[j].w & m[3]);
      // group i holds bits 8 (i % 4) .. 8 (i % 4) + 7 of keep word i / 4, and i % 4 == lane % 4
      uint32_t word = bits << (8 * (lane & 3));
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
      if (ok && (lane & 3) == 0) p.keep[i >> 2] = word;
    }
  }
}

// dx = bf16( base + s_d * keep * (v A) ): base = dy W_hat in fp32 from the
// GEMM, v = dy B [M, r], A [r, K].  A CTA owns 64 rows x 128 columns, warp w
// rows 16w..16w+15.  The base tile streams into shared memory by
// asynchronous copies issued first, while the thread loads its keep words
// and v A comes from the tensor cores (rank_tile_mma, accumulator layout:
// 2 rows x 32 columns per thread); each thread then adds s_d (v A) where
// its bit is set and rounds once.  HBM-bound: 4 + 1/8 bytes read and 2
// written per element; v and A come from L2.
struct DxDropoutParams {
  const float* base;          // [M, K]
  const uint32_t* keep;       // [M, K / 32]
  const __nv_bfloat16* v;     // [M, r]
  const __nv_bfloat16* A;     // [r, K]
  __nv_bfloat16* dx;          // [M, K]
  int64_t M, K;
  int r;                      // multiple of 8, >= 8
  float sd;                   // fl32(s / (1 - p))
};

// floats per staged base row: a half warp's 8-byte reads (4 rows x 32
// bytes) then fall in distinct banks
constexpr int kDxBasePitch = kTileCols + 8;

__host__ __device__ constexpr size_t dx_dropout_smem_bytes(int r) {
  return static_cast<size_t>(kTileRows) * kDxBasePitch * 4 + rank_tile_operand_bytes(r);
}

// 16-byte global -> shared copy that bypasses L1; src_bytes 0 writes zeros
// and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__global__ void __launch_bounds__(kTileThreads) lora_dx_dropout_kernel(DxDropoutParams p) {
  extern __shared__ __align__(16) uint8_t dxd_smem[];
  float* bs = reinterpret_cast<float*>(dxd_smem);                                         // [64][pitch]
  __nv_bfloat16* ops = reinterpret_cast<__nv_bfloat16*>(bs + kTileRows * kDxBasePitch);   // operands
  pdl_launch_dependents();
  pdl_wait_primary();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kTileRows;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kTileCols;

  // the base tile, 16 bytes per copy, zero past the last row or column
  for (int i = tid; i < kTileRows * (kTileCols / 4); i += kTileThreads) {
    const int row = i / (kTileCols / 4), c4 = (i % (kTileCols / 4)) * 4;
    const int64_t n = n0 + row, k = k0 + c4;
    const bool ok = n < p.M && k < p.K;
    cp_async16(smem_u32(bs + row * kDxBasePitch + c4), ok ? p.base + n * p.K + k : p.base, ok ? 16u : 0u);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");

  const int lrow[2] = {warp * 16 + g, warp * 16 + g + 8};
  const int64_t kw = p.K >> 5;
  // element (row, k0 + 8t + 2q + e): keep bit 8 (t % 4) + 2q + e of word kwd[h][t / 4]
  uint32_t kwd[2][4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t n = n0 + lrow[h];
#pragma unroll
    for (int w = 0; w < 4; ++w) kwd[h][w] = (n < p.M && k0 + 32 * w < p.K) ? p.keep[n * kw + (k0 >> 5) + w] : 0u;
  }
  float acc[16][4];
  rank_tile_mma(p.v, p.M, p.A, p.K, p.r, n0, k0, ops, acc);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t n = n0 + lrow[h];
    if (n >= p.M) continue;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const int cl = 8 * t + 2 * q;
      if (k0 + cl >= p.K) continue;
      const float2 b = *reinterpret_cast<const float2*>(bs + lrow[h] * kDxBasePitch + cl);
      const uint32_t bits = kwd[h][t >> 2] >> (8 * (t & 3) + 2 * q);
      const float o0 = __fadd_rn(b.x, (bits & 1u) ? __fmul_rn(p.sd, acc[t][2 * h]) : 0.f);
      const float o1 = __fadd_rn(b.y, (bits & 2u) ? __fmul_rn(p.sd, acc[t][2 * h + 1]) : 0.f);
      *reinterpret_cast<uint32_t*>(p.dx + n * p.K + k0 + cl) = pack_bf16x2(o0, o1);
    }
  }
}

}  // namespace qn
