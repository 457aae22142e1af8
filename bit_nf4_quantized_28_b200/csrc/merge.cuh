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
// are re-read from L2.  Persistent CTAs of 4 warps walk tiles of 64 rows x
// 128 columns; while a CTA works on one tile, asynchronous copies bring the
// next tile's codes, B rows and A columns into the other half of a double
// buffer, and its threads load the next tile's block scales into registers.
// Per tile:
//  1. warp w computes P = B A for rows 16w .. 16w + 15 on the tensor cores
//     (mma.sync m16n8k16, operands by ldmatrix), into registers;
//  2. each thread dequantizes the weights of its accumulator positions,
//     adds fl32(s P) and stores them.  A's columns are staged permuted so
//     that the MMA's column 8t + 2q + e is the tile's column
//     32 (t / 4) + 8q + 2 (t % 4) + e: a thread's accumulators of a row then
//     cover 8 consecutive columns per group of 32 (one 16-byte store, a
//     warp's store covering 64 contiguous bytes of each of 8 rows), and their
//     code bytes are one aligned 4-byte word of the row.
#pragma once

#include "common.cuh"
#include "lora_small.cuh"
#include "nf4_storage.cuh"

namespace qn {

constexpr int kMergeRows = 64;
constexpr int kMergeCols = 128;
constexpr int kMergeThreads = 128;
constexpr int kMergeRPad = kMergeCols + 8;   // bf16 per staged A row (ldmatrix without bank conflicts)

__host__ __device__ constexpr int merge_r16(int r) { return (r + 15) & ~15; }

// One buffer: codes [64][64 B], B rows [64][r16 + 8] bf16, A rows [r16][136] bf16.
__host__ __device__ constexpr size_t merge_buffer_bytes(int r) {
  return static_cast<size_t>(kMergeRows) * (kMergeCols / 2) +
         (r > 0 ? static_cast<size_t>(kMergeRows) * (merge_r16(r) + 8) * 2 +
                      static_cast<size_t>(merge_r16(r)) * kMergeRPad * 2
                : 0);
}
// The level table and two buffers.
__host__ __device__ constexpr size_t merge_smem_bytes(int r) { return 16 * 4 + 2 * merge_buffer_bytes(r); }

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Copies tile (n0, k0)'s codes, B rows and A columns into buffer `buf`
// (columns past K are not copied: the tile's valid columns are 128 or 64).
// A's column pair 16i + 4q + j (columns 32i + 8q + 2j, + 1) goes to staged
// pair 16i + 4j + q.
// A tile has 128 columns, or 64 (the last one when K % 128 == 64), so the
// per-row counts below are powers of two and the copies' row and column
// come from shifts; B's 16-byte chunks per row, r / 8 <= 16, come from an
// exact multiply-shift (i < 1024).
__device__ __forceinline__ void merge_stage(const MergeParams& p, int64_t n0, int64_t k0, int cols, uint8_t* buf) {
  const int tid = threadIdx.x;
  const int r = p.r, r16 = merge_r16(r);
  const uint32_t cs = smem_u32(buf);
  const int wide = cols == kMergeCols ? 1 : 0;
  // codes: 64 rows x cols / 2 bytes, 16 bytes per copy (2 << wide per row)
  const int cshift = 1 + wide;
  for (int i = tid; i < kMergeRows << cshift; i += kMergeThreads) {
    const int row = i >> cshift, c = i & ((1 << cshift) - 1);
    cp_async16(cs + row * (kMergeCols / 2) + c * 16, p.codes + (n0 + row) * (p.K >> 1) + (k0 >> 1) + c * 16);
  }
  if (r > 0) {
    const int lpad = r16 + 8;
    const uint32_t ls = cs + kMergeRows * (kMergeCols / 2);
    const uint32_t rs = ls + kMergeRows * lpad * 2;
    const int rc = r / 8;
    const uint32_t rmagic = (65536u + static_cast<uint32_t>(rc) - 1u) / static_cast<uint32_t>(rc);
    for (int i = tid; i < kMergeRows * rc; i += kMergeThreads) {
      const int row = static_cast<int>((static_cast<uint32_t>(i) * rmagic) >> 16), c8 = (i - row * rc) * 8;
      cp_async16(ls + (row * lpad + c8) * 2, p.B + (n0 + row) * r + c8);
    }
    const int pshift = 5 + wide;           // cols / 2 pairs of columns
    for (int i = tid; i < r << pshift; i += kMergeThreads) {
      const int j = i >> pshift, pr = i & ((1 << pshift) - 1);
      const int sp = (pr & ~15) | ((pr & 3) << 2) | ((pr >> 2) & 3);
      cp_async4(rs + (j * kMergeRPad + 2 * sp) * 2, p.A + static_cast<int64_t>(j) * p.K + k0 + 2 * pr);
    }
  }
}

// This thread's block scales of a tile: rows g and g + 8 of its warp's 16,
// blocks k0 / 64 and k0 / 64 + 1 (the second only if the tile has 128 columns).
struct MergeScales {
  int8_t q[2][2];
  float st[2][2], mn[2][2];
};
__device__ __forceinline__ void merge_load_scales(const MergeParams& p, int64_t n0, int64_t k0, int cols,
                                                  MergeScales& sc) {
  const int warp = threadIdx.x >> 5, g = (threadIdx.x & 31) >> 2;
  const int64_t kb = p.K >> 6;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int64_t blk = (n0 + warp * 16 + g + 8 * h) * kb + (k0 >> 6) + (b < cols / 64 ? b : 0);
      sc.q[h][b] = __ldg(p.qscale + blk);
      sc.st[h][b] = __ldg(p.dq_step + (blk >> 8));
      sc.mn[h][b] = __ldg(p.dq_mean + (blk >> 8));
    }
  }
}

__global__ void __launch_bounds__(kMergeThreads) qlora_merge_kernel(MergeParams p) {
  extern __shared__ __align__(16) uint8_t merge_smem[];
  const int r = p.r, r16 = merge_r16(r), lpad = r16 + 8;
  const size_t bufb = merge_buffer_bytes(r);
  float* lv = reinterpret_cast<float*>(merge_smem);                   // [16]
  uint8_t* bufs = merge_smem + 64;

  pdl_launch_dependents();
  pdl_wait_primary();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  if (tid < 16) lv[tid] = p.lv.v[tid];
  // zero the rank padding of both buffers once (B columns r .. r16 + 7, A rows r .. r16 - 1)
  if (r > 0 && r16 + 8 > r) {
    for (int bsel = 0; bsel < 2; ++bsel) {
      __nv_bfloat16* ls = reinterpret_cast<__nv_bfloat16*>(bufs + bsel * bufb + kMergeRows * (kMergeCols / 2));
      __nv_bfloat16* rs = ls + kMergeRows * lpad;
      for (int i = tid; i < kMergeRows * (lpad - r); i += kMergeThreads)
        ls[(i / (lpad - r)) * lpad + r + i % (lpad - r)] = __float2bfloat16_rn(0.f);
      for (int i = tid; i < (r16 - r) * kMergeRPad; i += kMergeThreads) rs[r * kMergeRPad + i] = __float2bfloat16_rn(0.f);
    }
  }

  // tiles run row-fastest, so that CTAs working at the same time share A's
  // columns in L2; a CTA's tiles are blockIdx.x, + gridDim.x, ..., walked as
  // (row tile, column tile) pairs without dividing
  const uint32_t ntr = static_cast<uint32_t>(p.N / kMergeRows);
  const uint32_t ntc = static_cast<uint32_t>((p.K + kMergeCols - 1) / kMergeCols);
  const uint32_t gq = gridDim.x / ntr, gr = gridDim.x % ntr;
  uint32_t tr = blockIdx.x % ntr, tcol = blockIdx.x / ntr;
  if (tcol >= ntc) return;
  auto coords = [&](uint32_t r_t, uint32_t c_t, int64_t& n0, int64_t& k0, int& cols) {
    n0 = static_cast<int64_t>(r_t) * kMergeRows;
    k0 = static_cast<int64_t>(c_t) * kMergeCols;
    cols = p.K - k0 < kMergeCols ? static_cast<int>(p.K - k0) : kMergeCols;
  };
  int64_t n0, k0;
  int cols;
  coords(tr, tcol, n0, k0, cols);
  merge_stage(p, n0, k0, cols, bufs);
  cp_async_commit();
  MergeScales sc;
  merge_load_scales(p, n0, k0, cols, sc);
  const float s = p.s;
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
      merge_stage(p, n1, k1, cols1, bufs + ((it + 1) & 1) * bufb);
    }
    cp_async_commit();
    cp_async_wait1();          // this tile's copies have landed
    __syncthreads();
    const uint8_t* buf = bufs + (it & 1) * bufb;
    const uint32_t cs = smem_u32(buf);
    // P = B A for the warp's 16 rows x 128 columns
    float acc[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    if (r > 0) {
      const uint32_t ls = cs + kMergeRows * (kMergeCols / 2);
      const uint32_t rs = ls + kMergeRows * lpad * 2;
      const int mi = lane >> 3, rr = lane & 7;
      for (int kk = 0; kk < r16; kk += 16) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(ls + ((warp * 16 + (mi & 1) * 8 + rr) * lpad + kk + (mi >> 1) * 8) * 2, a0, a1, a2, a3);
#pragma unroll
        for (int t = 0; t < 16; t += 2) {
          if (8 * t >= cols) break;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(rs + ((kk + (mi & 1) * 8 + rr) * kMergeRPad + 8 * t + (mi >> 1) * 8) * 2, b0, b1, b2, b3);
          mma_bf16_16816(acc[t], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    // the next tile's scales (their loads overlap the work below)
    MergeScales sc1 = sc;
    if (more) merge_load_scales(p, n1, k1, cols1, sc1);
    // dequantize, add fl32(s P), store: row g (h = 0) and g + 8 (h = 1),
    // columns 32i + 8q .. + 7 from accumulators t = 4i .. 4i + 3
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = warp * 16 + g + 8 * h;
      const float sh0 = restore_scale(sc.q[h][0], sc.st[h][0], sc.mn[h][0]);
      const float sh1 = restore_scale(sc.q[h][1], sc.st[h][1], sc.mn[h][1]);
      __nv_bfloat16* orow = p.out + (n0 + row) * p.K + k0 + 8 * q;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (32 * i >= cols) break;
        // bytes 16i + 4q .. + 3 of the row: byte j holds columns 32i + 8q + 2j, + 1
        const uint32_t cw = *reinterpret_cast<const uint32_t*>(buf + row * (kMergeCols / 2) + 16 * i + 4 * q);
        const float sh = i < 2 ? sh0 : sh1;
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = 4 * i + j;
          const uint32_t c = (cw >> (8 * j)) & 0xFFu;
          const float w0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[c & 15u], sh)));
          const float w1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[c >> 4], sh)));
          const float e0 = r > 0 ? __fmul_rn(s, acc[t][2 * h]) : 0.f;
          const float e1 = r > 0 ? __fmul_rn(s, acc[t][2 * h + 1]) : 0.f;
          o[j] = pack_bf16x2(__fadd_rn(w0, e0), __fadd_rn(w1, e1));
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
    sc = sc1;
  }
}

}  // namespace qn
