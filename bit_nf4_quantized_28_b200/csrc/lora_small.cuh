// lora_small.cuh -- the rank-r products of the LoRA path.
//
// [skyvanguard "LoRA y QLoRA en Profundidad", "Cómo Funciona LoRA": A is
//  (r x d_in), B is (d_out x r); "Alpha (lora_alpha)": scale alpha / r.
//  QLoRA glossary, "Come funziona QLoRA": the LoRA output is added to the
//  frozen path; backpropagation updates only the two LoRA matrices.]
//
//   down:  P[m][j] = sum_k X[m][k] * W(j, k)        (u = x A^T, v = dy B)
//   up:    P[p][j] = sum_m X[m][p] * V[m][j]        (dA^T = x^T v, dB = dy^T u)
//
// These are HBM-bound (reading x or dy once), so they use mma.sync
// m16n8k16 bf16 tiles staged through shared memory.  Work is split over
// the reduction dimension into fixed chunks; each chunk writes an fp32
// partial and a finalize kernel sums the partials in a fixed order, so the
// result does not depend on scheduling.
#pragma once

#include "common.cuh"

namespace qn {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int kSmallTile = 64;     // rows of the output tile per CTA and reduction step
constexpr int kSmallPad = 72;      // padded smem row length (bf16), breaks bank conflicts
constexpr int kMaxRank = 128;

// One rank-r product.  `kind` 0 = down, 1 = up.
struct SmallProblem {
  int kind;
  const __nv_bfloat16* X;   // down: [rows, red] ; up: [red, rows]
  const __nv_bfloat16* W;   // down: W(j, k) ; up: V [red, r]
  int w_transposed;         // down only: 0 -> W[j*red + k], 1 -> W[k*r + j]
  int64_t rows;             // output rows (M for down, P for up)
  int64_t red;              // reduction length (K for down, M for up)
  int r;
  int64_t chunk;            // reduction chunk per split (multiple of 64)
  int splits;
  int tiles;                // ceil(rows / 64)
  float* partial;           // [splits][rows][r] fp32
};

struct SmallBatch {
  SmallProblem p[2];
  int count;
  int blocks0;              // CTAs of problem 0 (tiles * splits)
};

// 128 threads: warp w owns output rows [16w, 16w + 16) of the 64-row tile.
__global__ void __launch_bounds__(128) lora_partial_kernel(SmallBatch batch) {
  __shared__ __align__(16) __nv_bfloat16 sX[kSmallTile][kSmallPad];
  __shared__ __align__(16) __nv_bfloat16 sW[kMaxRank][kSmallPad];
  pdl_launch_dependents();
  int bid = blockIdx.x;
  const int pi = (batch.count > 1 && bid >= batch.blocks0) ? 1 : 0;
  if (pi) bid -= batch.blocks0;
  const SmallProblem& P = batch.p[pi];
  const int tile = bid % P.tiles;
  const int split = bid / P.tiles;
  const int64_t row0 = static_cast<int64_t>(tile) * kSmallTile;
  const int64_t k_begin = static_cast<int64_t>(split) * P.chunk;
  int64_t k_end = k_begin + P.chunk;
  if (k_end > P.red) k_end = P.red;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int r = P.r, nt = r >> 3;

  // The inputs of this kernel may be written by the preceding kernel.
  pdl_wait_primary();

  float acc[kMaxRank / 8][4];
#pragma unroll
  for (int t = 0; t < kMaxRank / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  for (int64_t k0 = k_begin; k0 < k_end; k0 += kSmallTile) {
    __syncthreads();
    if (P.kind == 0) {
      // sX[m][k] = X[row0 + m][k0 + k]; rows past the end are zero.
      for (int i = tid; i < kSmallTile * 8; i += 128) {
        const int m = i >> 3, c = (i & 7) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row0 + m < P.rows && k0 + c < k_end)
          v = *reinterpret_cast<const uint4*>(P.X + (row0 + m) * P.red + k0 + c);
        *reinterpret_cast<uint4*>(&sX[m][c]) = v;
      }
      // sW[j][k] = W(j, k0 + k)
      if (!P.w_transposed) {
        for (int i = tid; i < r * 8; i += 128) {
          const int j = i >> 3, c = (i & 7) * 8;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (k0 + c < k_end) v = *reinterpret_cast<const uint4*>(P.W + j * P.red + k0 + c);
          *reinterpret_cast<uint4*>(&sW[j][c]) = v;
        }
      } else {
        const int per_row = r >> 3;   // uint4 per source row (8 bf16 each)
        for (int i = tid; i < kSmallTile * per_row; i += 128) {
          const int k = i / per_row, jc = (i % per_row) * 8;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (k0 + k < k_end) v = *reinterpret_cast<const uint4*>(P.W + (k0 + k) * r + jc);
          const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
          for (int u = 0; u < 8; ++u) sW[jc + u][k] = e[u];
        }
      }
    } else {
      // up: sX[p][m] = X[k0 + m][row0 + p]  (transposed), sW[j][m] = V[k0 + m][j]
      for (int i = tid; i < kSmallTile * 8; i += 128) {
        const int m = i >> 3, c = (i & 7) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (k0 + m < k_end && row0 + c < P.rows)
          v = *reinterpret_cast<const uint4*>(P.X + (k0 + m) * P.rows + row0 + c);
        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
        for (int u = 0; u < 8; ++u) sX[c + u][m] = e[u];
      }
      const int per_row = r >> 3;
      for (int i = tid; i < kSmallTile * per_row; i += 128) {
        const int m = i / per_row, jc = (i % per_row) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (k0 + m < k_end) v = *reinterpret_cast<const uint4*>(P.W + (k0 + m) * r + jc);
        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
        for (int u = 0; u < 8; ++u) sW[jc + u][m] = e[u];
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSmallTile; kk += 16) {
      const int ra = warp * 16 + g;
      const uint32_t a0 = *reinterpret_cast<const uint32_t*>(&sX[ra][kk + 2 * q]);
      const uint32_t a1 = *reinterpret_cast<const uint32_t*>(&sX[ra + 8][kk + 2 * q]);
      const uint32_t a2 = *reinterpret_cast<const uint32_t*>(&sX[ra][kk + 2 * q + 8]);
      const uint32_t a3 = *reinterpret_cast<const uint32_t*>(&sX[ra + 8][kk + 2 * q + 8]);
#pragma unroll
      for (int t = 0; t < kMaxRank / 8; ++t) {
        if (t < nt) {
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&sW[8 * t + g][kk + 2 * q]);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&sW[8 * t + g][kk + 2 * q + 8]);
          mma_bf16_16816(acc[t], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
  // partial[split][row][j]
  float* out = P.partial + static_cast<int64_t>(split) * P.rows * r;
  const int64_t rr = row0 + warp * 16 + g;
#pragma unroll
  for (int t = 0; t < kMaxRank / 8; ++t) {
    if (t < nt) {
      const int j = 8 * t + 2 * q;
      if (rr < P.rows) *reinterpret_cast<float2*>(out + rr * r + j) = make_float2(acc[t][0], acc[t][1]);
      if (rr + 8 < P.rows)
        *reinterpret_cast<float2*>(out + (rr + 8) * r + j) = make_float2(acc[t][2], acc[t][3]);
    }
  }
}

// Finalize of a down product: sums the partials in split order and writes
//   plain  bf16 [rows, r]  = bf16(sum)             (if non-null)
//   scaled bf16 [rows, rp] = bf16(fl32(s * sum)), zero for j >= r (if non-null)
// Finalize of an up product: out fp32 = fl32(s * sum), stored [rows, r]
// or transposed [r, rows].
struct SmallFinal {
  const float* partial;
  int64_t rows;
  int r;
  int splits;
  float s;
  int kind;                  // 0 = down, 1 = up
  __nv_bfloat16* plain;      // down
  __nv_bfloat16* scaled;     // down
  int rp;                    // down: padded width of `scaled`
  float* out;                // up
  int transpose;             // up: 1 -> out[j*rows + p]
};

struct SmallFinalBatch {
  SmallFinal f[2];
  int count;
  int64_t items0;            // threads' work items of f[0]
};

__global__ void __launch_bounds__(256) lora_finalize_kernel(SmallFinalBatch b) {
  pdl_launch_dependents();
  pdl_wait_primary();
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  int fi = 0;
  if (b.count > 1 && i >= b.items0) {
    fi = 1;
    i -= b.items0;
  }
  const SmallFinal& F = b.f[fi];
  if (F.kind == 0) {
    // one item per (row, padded column)
    const int64_t row = i / F.rp;
    const int j = static_cast<int>(i % F.rp);
    if (row >= F.rows) return;
    float sum = 0.f;
    if (j < F.r)
      for (int s = 0; s < F.splits; ++s) sum += F.partial[(static_cast<int64_t>(s) * F.rows + row) * F.r + j];
    if (F.plain && j < F.r) F.plain[row * F.r + j] = __float2bfloat16_rn(sum);
    if (F.scaled) F.scaled[row * F.rp + j] = __float2bfloat16_rn(j < F.r ? __fmul_rn(F.s, sum) : 0.f);
  } else {
    const int64_t row = i / F.r;
    const int j = static_cast<int>(i % F.r);
    if (row >= F.rows) return;
    float sum = 0.f;
    for (int s = 0; s < F.splits; ++s) sum += F.partial[(static_cast<int64_t>(s) * F.rows + row) * F.r + j];
    const float v = __fmul_rn(F.s, sum);
    if (F.transpose) F.out[static_cast<int64_t>(j) * F.rows + row] = v;
    else F.out[row * F.r + j] = v;
  }
}

}  // namespace qn
