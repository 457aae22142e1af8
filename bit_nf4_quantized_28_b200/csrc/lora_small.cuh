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
// These are HBM-bound (each reads x or dy once), so the tiles use mma.sync
// m16n8k16 on bf16, fed by a cp.async ring and ldmatrix.  One output tile
// (64 rows x a range of rank columns) belongs to a thread-block cluster: the
// cluster's CTAs split the reduction dimension, park their fp32 partial tile
// in their own shared memory, and each CTA then sums one slice of the tile
// over distributed shared memory, in rank order, and writes it.  No
// partial leaves the chip, there is one launch per product, and the sum's
// order is fixed, so results are reproducible.
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

constexpr int kSmallTile = 64;     // output rows per tile and reduction step length
constexpr int kSmallPad = 72;      // padded smem row of a 64-wide tile (bf16): conflict-free ldmatrix
constexpr int kMaxRank = 128;
constexpr int kClusterStages = 4;       // ring depth, one cluster per tile
constexpr int kPersistStages = 8;       // ring depth, persistent CTAs
constexpr int kMaxCluster = 8;

// One rank-r product.  `kind` 0 = down, 1 = up.
struct SmallProblem {
  int kind;
  const __nv_bfloat16* X;   // down: [rows, red] ; up: [red, rows]
  const __nv_bfloat16* W;   // down: W(j, k) ; up: V [red, r]
  int w_transposed;         // down only: 0 -> W[j*red + k], 1 -> W[k*r + j]
  int64_t rows;             // output rows (M for down, P for up)
  int64_t red;              // reduction length (K for down, M for up)
  int r;
  int rj;                   // rank columns per tile (r / column splits, multiple of 16 or r)
  int csplit;               // column splits
  int64_t chunk;            // reduction elements per CTA of a cluster (multiple of 64)
  int tiles;                // ceil(rows / 64)
  float s;                  // output scale
  // down outputs
  __nv_bfloat16* plain;     // [rows, r] bf16(sum), or null
  __nv_bfloat16* scaled;    // [rows, rp] bf16(fl32(s * sum)), zero padded, or null
  int rp;
  // up output
  float* out;               // fl32(s * sum): [rows, r], or [r, rows] when transpose
  int transpose;
};

struct SmallBatch {
  SmallProblem p[2];
  int count;
  int clusters0;            // clusters of problem 0 (tiles * csplit)
  int clusters;             // clusters of all problems
  int cs;                   // CTAs per cluster (reduction splits)
  int w_stride;             // padded row length of the rank-side tile (elements)
  int w_tile_elems;         // elements of one stage's rank-side tile
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_cluster(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// 128 threads: warp w owns output rows [16w, 16w + 16) of the 64-row tile and
// the tile's rj = 8 * NT rank columns.  Launched with cluster size batch.cs.
// Two ways to launch it: one cluster per tile, with the cluster splitting
// the reduction (a short kernel over the whole GPU); or a few persistent
// CTAs (cs = 1) that walk the tiles, each tile reduced by one CTA, sized to
// run on the SMs the tensor-core GEMM that follows leaves free.  The code is
// kept compact (the k16 loop stays rolled; NT and the ring depth are
// template parameters) to limit cold instruction-cache misses.
template <int NT, int kSmallStages>
__global__ void __launch_bounds__(128) lora_rank_kernel(SmallBatch batch) {
  extern __shared__ __align__(16) __nv_bfloat16 small_smem[];
  pdl_launch_dependents();
  // The inputs of this kernel may be written by the preceding kernel.
  pdl_wait_primary();
  const int cs = batch.cs;
  const int q_rank = static_cast<int>(cluster_rank());
  for (int clg = blockIdx.x / cs; clg < batch.clusters; clg += gridDim.x / cs) {
  int cl = clg;
  const int pi = (batch.count > 1 && cl >= batch.clusters0) ? 1 : 0;
  if (pi) cl -= batch.clusters0;
  const SmallProblem P = batch.p[pi];          // by value: fields live in registers
  const int tile = cl % P.tiles;
  const int csp = cl / P.tiles;
  const int j0 = csp * P.rj;
  const int64_t row0 = static_cast<int64_t>(tile) * kSmallTile;
  const int64_t k_begin = static_cast<int64_t>(q_rank) * P.chunk;
  int64_t k_end = k_begin + P.chunk;
  if (k_end > P.red) k_end = P.red;
  const int nsteps = k_end > k_begin ? static_cast<int>((k_end - k_begin + kSmallTile - 1) / kSmallTile) : 0;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int r = P.r, rj = P.rj;
  constexpr int nt = NT;
  const int ws = batch.w_stride;
  const int x_elems = kSmallTile * kSmallPad;
  const int stage_elems = x_elems + batch.w_tile_elems;
  const uint32_t smem0 = smem_u32(small_smem);
  const int kind = P.kind, wtr = P.w_transposed;

  // Copy assignments, fixed for the whole loop: each thread moves four
  // 16-byte chunks of the 64 x 64 X tile (rows xr + 16 i, column chunk xc)
  // and up to NT chunks of the rank-side tile; per step only the reduction
  // offset advances.
  const int xr = tid >> 3, xc = (tid & 7) * 8;
  const __nv_bfloat16* xsrc[4];
  bool xrow_ok[4];
  uint32_t xdst[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = xr + 16 * i;
    xdst[i] = static_cast<uint32_t>((m * kSmallPad + xc) * 2);
    if (kind == 0) {
      // down: sX[m][k] = X[row0 + m][k_begin + k]; the reduction runs along the row
      xrow_ok[i] = row0 + m < P.rows;
      xsrc[i] = P.X + (xrow_ok[i] ? (row0 + m) * P.red + k_begin + xc : 0);
    } else {
      // up: sX[m][p] = X[k_begin + m][row0 + p]; the reduction runs down the rows
      xrow_ok[i] = row0 + xc < P.rows;
      xsrc[i] = P.X + (xrow_ok[i] ? (k_begin + m) * P.rows + row0 + xc : 0);
    }
  }
  const int64_t x_step = kind == 0 ? kSmallTile : kSmallTile * P.rows;   // elements per reduction step
  // rank-side chunks: non-transposed W: rj rows x 8 chunks; otherwise 64 rows x rj/8 chunks
  const int wper = (kind == 0 && !wtr) ? 8 : (rj >> 3);
  const int wchunks = (kind == 0 && !wtr) ? rj * 8 : kSmallTile * wper;
  const int64_t w_step = (kind == 0 && !wtr) ? kSmallTile : static_cast<int64_t>(kSmallTile) * r;

  auto load_stage = [&](int step, int stage) {
    const int64_t kofs = static_cast<int64_t>(step) * kSmallTile;     // reduction offset within the chunk
    const uint32_t sx = smem0 + static_cast<uint32_t>(stage * stage_elems) * 2;
    const uint32_t sw = sx + x_elems * 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // k-bound: down checks the column chunk, up checks the row
      const bool kin = kind == 0 ? (k_begin + kofs + xc < k_end) : (k_begin + kofs + xr + 16 * i < k_end);
      const bool ok = xrow_ok[i] && kin;
      cp_async16(sx + xdst[i], ok ? xsrc[i] + step * x_step : P.X, ok);
    }
    for (int c = tid; c < wchunks; c += 128) {
      const int a = c / wper, b = (c % wper) * 8;      // a: smem row, b: column (elements)
      bool ok;
      const __nv_bfloat16* src;
      uint32_t dst;
      if (kind == 0 && !wtr) {
        // sW[j][k] = W[j0 + j][k_begin + kofs + k]
        ok = k_begin + kofs + b < k_end;
        src = P.W + (j0 + a) * P.red + k_begin + kofs + b;
        dst = static_cast<uint32_t>((a * kSmallPad + b) * 2);
      } else {
        // sW[k][j] = W[k_begin + kofs + k][j0 + j]  (also V for the up products)
        ok = k_begin + kofs + a < k_end;
        src = P.W + (k_begin + kofs + a) * r + j0 + b;
        dst = static_cast<uint32_t>((a * ws + b) * 2);
      }
      cp_async16(sw + dst, ok ? src : P.W, ok);
    }
    (void)w_step;
  };

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

#pragma unroll
  for (int s = 0; s < kSmallStages - 1; ++s) {
    if (s < nsteps) load_stage(s, s);
    cp_async_commit();
  }
  // ldmatrix lane roles: matrix mi = lane / 8, row rr = lane % 8 of it
  const int mi = lane >> 3, rr = lane & 7;
  for (int step = 0; step < nsteps; ++step) {
    cp_async_wait<kSmallStages - 2>();
    __syncthreads();
    {
      const int nxt = step + kSmallStages - 1;
      if (nxt < nsteps) load_stage(nxt, nxt % kSmallStages);
      cp_async_commit();
    }
    const int stage = step % kSmallStages;
    const uint32_t sx = smem0 + static_cast<uint32_t>(stage * stage_elems) * 2;
    const uint32_t sw = sx + x_elems * 2;
#pragma unroll 1
    for (int kk = 0; kk < kSmallTile; kk += 16) {
      uint32_t a0, a1, a2, a3;
      if (kind == 0) {
        // A[m][k] = sX[m][k]: matrices (m 0-7, k 0-7), (m 8-15, k 0-7), (m 0-7, k 8-15), (m 8-15, k 8-15)
        const int m = warp * 16 + (mi & 1) * 8 + rr, k = kk + (mi >> 1) * 8;
        ldsm_x4(sx + (m * kSmallPad + k) * 2, a0, a1, a2, a3);
      } else {
        // A[p][m] = sX[m][p] (transposed load)
        const int m = kk + (mi >> 1) * 8 + rr, pcol = warp * 16 + (mi & 1) * 8;
        ldsm_x4_t(sx + (m * kSmallPad + pcol) * 2, a0, a1, a2, a3);
      }
#pragma unroll
      for (int t = 0; t < NT; t += 2) {
        {
          uint32_t b0, b1, b2, b3;
          if (kind == 0 && !wtr) {
            // B[k][j] = sW[j][k]: matrices (j 0-7, k 0-7), (j 0-7, k 8-15), (j 8-15, k 0-7), (j 8-15, k 8-15)
            const int j = 8 * t + (mi >> 1) * 8 + rr, k = kk + (mi & 1) * 8;
            ldsm_x4(sw + (j * kSmallPad + k) * 2, b0, b1, b2, b3);
          } else {
            // B[k][j] = sW[k][j] (transposed load): (k 0-7, j 0-7), (k 8-15, j 0-7), (k 0-7, j 8-15), (k 8-15, j 8-15)
            const int k = kk + (mi & 1) * 8 + rr, j = 8 * t + (mi >> 1) * 8;
            ldsm_x4_t(sw + (k * ws + j) * 2, b0, b1, b2, b3);
          }
          mma_bf16_16816(acc[t], a0, a1, a2, a3, b0, b1);
          if (t + 1 < nt) mma_bf16_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // This CTA's partial tile: red[row][j] fp32 at the start of shared memory.
  float* red = reinterpret_cast<float*>(small_smem);
  {
    const int ro = warp * 16 + g;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      {
        const int j = 8 * t + 2 * q;
        red[ro * rj + j] = acc[t][0];
        red[ro * rj + j + 1] = acc[t][1];
        red[(ro + 8) * rj + j] = acc[t][2];
        red[(ro + 8) * rj + j + 1] = acc[t][3];
      }
    }
  }
  cluster_sync_all();
  // Every CTA of the cluster reduces its own slice of the tile: groups of
  // four partial values are read from all cs CTAs first, then added in rank
  // order (a fixed order, so the result is reproducible).
  {
    const uint32_t red0 = smem_u32(red);
    const int nvec = kSmallTile * rj / 4;
    const int per = (nvec + cs - 1) / cs;
    const int v0 = q_rank * per;
    const int v1 = min(nvec, v0 + per);
    for (int v = v0 + tid; v < v1; v += 128) {
      float4 part[kMaxCluster];
#pragma unroll
      for (int c = 0; c < kMaxCluster; ++c)
        if (c < cs) part[c] = ld_cluster_f32x4(map_cluster(red0 + 16u * v, c));
      float4 sum = part[0];
#pragma unroll
      for (int c = 1; c < kMaxCluster; ++c) {
        if (c < cs) {
          sum.x += part[c].x; sum.y += part[c].y; sum.z += part[c].z; sum.w += part[c].w;
        }
      }
      const int lr = (4 * v) / rj, j = (4 * v) % rj;
      const int64_t row = row0 + lr;
      if (row >= P.rows) continue;
      const int jj = j0 + j;
      const float e[4] = {sum.x, sum.y, sum.z, sum.w};
      if (P.kind == 0) {
        if (P.plain) {
#pragma unroll
          for (int u = 0; u < 4; ++u) P.plain[row * r + jj + u] = __float2bfloat16_rn(e[u]);
        }
        if (P.scaled) {
#pragma unroll
          for (int u = 0; u < 4; ++u) P.scaled[row * P.rp + jj + u] = __float2bfloat16_rn(__fmul_rn(P.s, e[u]));
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float val = __fmul_rn(P.s, e[u]);
          if (P.transpose) P.out[static_cast<int64_t>(jj + u) * P.rows + row] = val;
          else P.out[row * r + jj + u] = val;
        }
      }
    }
    // zero padding of the scaled copy past rank r (written once, by column split 0)
    if (P.kind == 0 && P.scaled && csp == 0 && q_rank == 0) {
      const int pad = P.rp - r;
      for (int i = tid; i < kSmallTile * pad; i += 128) {
        const int64_t row = row0 + i / pad;
        if (row < P.rows) P.scaled[row * P.rp + r + i % pad] = __float2bfloat16_rn(0.f);
      }
    }
  }
  // Keep every CTA's shared memory alive until all CTAs have read it (and,
  // with one CTA per cluster, finish with it before the next tile reuses it).
  cluster_sync_all();
  }
}

}  // namespace qn
