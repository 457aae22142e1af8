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
#include "merge.cuh"

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
// GEMM, v = dy B [M, r], A [r, K].  HBM-bound: 4 + 1/8 bytes read and 2
// written per element; v and A come from L2.  Persistent CTAs of 4 warps
// walk tiles of 64 rows x 64 columns (row-fastest, so that the CTAs working
// at the same time share A's columns in L2); while a CTA works on one tile,
// asynchronous copies bring the next tile's base, v rows and A columns into
// the other half of a double buffer, and its threads load the next tile's
// keep words into registers.  Per tile, warp w computes P = v A for rows
// 16w .. 16w + 15 on the tensor cores (mma.sync, as the LoRA merge does,
// with A's columns staged permuted so that a thread's accumulators of a row
// cover 8 consecutive columns per group of 32); each thread then reads those
// 8 columns of base (two 16-byte loads), adds s_d P where its keep bit is
// set, rounds once and writes them with one 16-byte store.
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

constexpr int kDxRows = 64;
constexpr int kDxCols = 64;                  // K is a multiple of 64: every tile is whole
constexpr int kDxRPad = kDxCols + 8;         // bf16 per staged A row (ldmatrix without bank conflicts)
constexpr int kDxT = kDxCols / 8;            // accumulator tiles of 8 columns per warp
constexpr int kDxThreads = 128;

// One buffer: base [64][64] fp32 (16-byte chunk c of row y at chunk
// c ^ (y & 1), so that a quarter warp's 16-byte reads of rows 2k and 2k + 1
// fall in distinct banks), v rows [64][r16 + 8] bf16, A [r16][72] bf16.  At
// rank 16 a buffer is 21.4 KB and four CTAs fit per SM.
__host__ __device__ constexpr size_t dx_buffer_bytes(int r) {
  return static_cast<size_t>(kDxRows) * kDxCols * 4 + static_cast<size_t>(kDxRows) * (merge_r16(r) + 8) * 2 +
         static_cast<size_t>(merge_r16(r)) * kDxRPad * 2;
}
__host__ __device__ constexpr size_t dx_dropout_smem_bytes(int r) { return 2 * dx_buffer_bytes(r); }

// Copies tile (n0, k0)'s base, v rows and A columns into buffer `buf` (rows
// past M are not copied: their outputs are not written).
__device__ __forceinline__ void dx_stage(const DxDropoutParams& p, int64_t n0, int64_t k0, int cols, uint8_t* buf) {
  const int tid = threadIdx.x;
  const int r = p.r, r16 = merge_r16(r), lpad = r16 + 8;
  const uint32_t bs = smem_u32(buf);
  (void)cols;
  // base: 64 rows x 16 chunks of 16 bytes
  constexpr int cshift = 4;
  for (int i = tid; i < kDxRows << cshift; i += kDxThreads) {
    const int row = i >> cshift, c = i & ((1 << cshift) - 1);
    if (n0 + row < p.M)
      cp_async16(bs + row * (kDxCols * 4) + ((c ^ (row & 1)) << 4), p.base + (n0 + row) * p.K + k0 + 4 * c);
  }
  const uint32_t ls = bs + kDxRows * kDxCols * 4;
  const uint32_t rs = ls + kDxRows * lpad * 2;
  const int rc = r / 8;
  const uint32_t rmagic = (65536u + static_cast<uint32_t>(rc) - 1u) / static_cast<uint32_t>(rc);
  for (int i = tid; i < kDxRows * rc; i += kDxThreads) {
    const int row = static_cast<int>((static_cast<uint32_t>(i) * rmagic) >> 16), c8 = (i - row * rc) * 8;
    if (n0 + row < p.M) cp_async16(ls + (row * lpad + c8) * 2, p.v + (n0 + row) * r + c8);
  }
  // A's column pair 16i + 4q + j (columns 32i + 8q + 2j, + 1) goes to staged pair 16i + 4j + q
  constexpr int pshift = 5;              // 32 pairs of columns
  for (int i = tid; i < r << pshift; i += kDxThreads) {
    const int j = i >> pshift, pr = i & ((1 << pshift) - 1);
    const int sp = (pr & ~15) | ((pr & 3) << 2) | ((pr >> 2) & 3);
    cp_async4(rs + (j * kDxRPad + 2 * sp) * 2, p.A + static_cast<int64_t>(j) * p.K + k0 + 2 * pr);
  }
}

// This thread's keep words of a tile: rows g and g + 8 of its warp's 16,
// column groups 0 and 1 (zero past M).
__device__ __forceinline__ void dx_load_keep(const DxDropoutParams& p, int64_t n0, int64_t k0, int cols,
                                             uint32_t (&kw)[2][kDxCols / 32]) {
  (void)cols;
  const int warp = threadIdx.x >> 5, g = (threadIdx.x & 31) >> 2;
  const int64_t kwr = p.K >> 5;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t n = n0 + warp * 16 + g + 8 * h;
#pragma unroll
    for (int i = 0; i < kDxCols / 32; ++i) kw[h][i] = (n < p.M) ? __ldg(p.keep + n * kwr + (k0 >> 5) + i) : 0u;
  }
}

__global__ void __launch_bounds__(kDxThreads) lora_dx_dropout_kernel(DxDropoutParams p) {
  extern __shared__ __align__(16) uint8_t dxd_smem[];
  const int r = p.r, r16 = merge_r16(r), lpad = r16 + 8;
  const size_t bufb = dx_buffer_bytes(r);
  pdl_launch_dependents();
  pdl_wait_primary();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  // zero the rank padding of both buffers once (v columns r .. r16 + 7, A rows r .. r16 - 1)
  if (r16 + 8 > r) {
    for (int bsel = 0; bsel < 2; ++bsel) {
      __nv_bfloat16* ls = reinterpret_cast<__nv_bfloat16*>(dxd_smem + bsel * bufb + kDxRows * kDxCols * 4);
      __nv_bfloat16* rs = ls + kDxRows * lpad;
      for (int i = tid; i < kDxRows * (lpad - r); i += kDxThreads)
        ls[(i / (lpad - r)) * lpad + r + i % (lpad - r)] = __float2bfloat16_rn(0.f);
      for (int i = tid; i < (r16 - r) * kDxRPad; i += kDxThreads) rs[r * kDxRPad + i] = __float2bfloat16_rn(0.f);
    }
  }
  // tiles run row-fastest; a CTA's tiles are blockIdx.x, + gridDim.x, ...,
  // walked as (row tile, column tile) pairs without dividing
  const uint32_t ntr = static_cast<uint32_t>((p.M + kDxRows - 1) / kDxRows);
  const uint32_t ntc = static_cast<uint32_t>((p.K + kDxCols - 1) / kDxCols);
  const uint32_t gq = gridDim.x / ntr, gr = gridDim.x % ntr;
  uint32_t tr = blockIdx.x % ntr, tcol = blockIdx.x / ntr;
  if (tcol >= ntc) return;
  auto coords = [&](uint32_t r_t, uint32_t c_t, int64_t& n0, int64_t& k0, int& cols) {
    n0 = static_cast<int64_t>(r_t) * kDxRows;
    k0 = static_cast<int64_t>(c_t) * kDxCols;
    cols = p.K - k0 < kDxCols ? static_cast<int>(p.K - k0) : kDxCols;
  };
  int64_t n0, k0;
  int cols;
  coords(tr, tcol, n0, k0, cols);
  dx_stage(p, n0, k0, cols, dxd_smem);
  cp_async_commit();
  uint32_t kw[2][kDxCols / 32];
  dx_load_keep(p, n0, k0, cols, kw);
  const float sd = p.sd;
  for (int it = 0;; ++it) {
    uint32_t tr1 = tr + gr, tc1 = tcol + gq;
    if (tr1 >= ntr) {
      tr1 -= ntr;
      ++tc1;
    }
    const bool more = tc1 < ntc;
    int64_t n1 = 0, k1 = 0;
    int cols1 = 0;
    if (more) {
      coords(tr1, tc1, n1, k1, cols1);
      dx_stage(p, n1, k1, cols1, dxd_smem + ((it + 1) & 1) * bufb);
    }
    cp_async_commit();
    cp_async_wait1();          // this tile's copies have landed
    __syncthreads();
    const uint8_t* buf = dxd_smem + (it & 1) * bufb;
    const uint32_t bs = smem_u32(buf);
    // P = v A for the warp's 16 rows x 64 columns
    float acc[kDxT][4];
#pragma unroll
    for (int t = 0; t < kDxT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    {
      const uint32_t ls = bs + kDxRows * kDxCols * 4;
      const uint32_t rs = ls + kDxRows * lpad * 2;
      const int mi = lane >> 3, rr = lane & 7;
      for (int kk = 0; kk < r16; kk += 16) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(ls + ((warp * 16 + (mi & 1) * 8 + rr) * lpad + kk + (mi >> 1) * 8) * 2, a0, a1, a2, a3);
#pragma unroll
        for (int t = 0; t < kDxT; t += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(rs + ((kk + (mi & 1) * 8 + rr) * kDxRPad + 8 * t + (mi >> 1) * 8) * 2, b0, b1, b2, b3);
          mma_bf16_16816(acc[t], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    // the next tile's keep words (their loads overlap the work below)
    uint32_t kw1[2][kDxCols / 32];
    if (more) dx_load_keep(p, n1, k1, cols1, kw1);
    // add s_d P where kept, round once, store: row g (h = 0) and g + 8
    // (h = 1), columns 32i + 8q .. + 7 from accumulators t = 4i .. 4i + 3
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = warp * 16 + g + 8 * h;
      if (n0 + row >= p.M) continue;
      __nv_bfloat16* orow = p.dx + (n0 + row) * p.K + k0 + 8 * q;
      const uint32_t brow = bs + row * (kDxCols * 4);
#pragma unroll
      for (int i = 0; i < kDxCols / 32; ++i) {
        const int c0 = 8 * i + 2 * q;
        const float4 ba = ld_shared_f4_v(brow + ((c0 ^ (row & 1)) << 4));
        const float4 bb = ld_shared_f4_v(brow + (((c0 + 1) ^ (row & 1)) << 4));
        const float b[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
        const uint32_t bits = kw[h][i] >> (8 * q);
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = 4 * i + j;
          const float o0 = __fadd_rn(b[2 * j], ((bits >> (2 * j)) & 1u) ? __fmul_rn(sd, acc[t][2 * h]) : 0.f);
          const float o1 = __fadd_rn(b[2 * j + 1], ((bits >> (2 * j + 1)) & 1u) ? __fmul_rn(sd, acc[t][2 * h + 1]) : 0.f);
          o[j] = pack_bf16x2(o0, o1);
        }
        *reinterpret_cast<uint4*>(orow + 32 * i) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    if (!more) break;
    __syncthreads();           // this buffer is refilled by the copy issued next iteration
    tr = tr1;
    tcol = tc1;
    n0 = n1;
    k0 = k1;
    cols = cols1;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < kDxCols / 32; ++i) kw[h][i] = kw1[h][i];
  }
}

}  // namespace qn
