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
// m16n8k16 on bf16, fed by a TMA ring of 128-byte-swizzled 64 x 64 boxes and
// ldmatrix (transposed where an operand is stored the other way round).  One output tile
// (64 rows x a range of rank columns) belongs to a thread-block cluster: the
// cluster's CTAs split the reduction dimension, park their fp32 partial tile
// in their own shared memory, and each CTA then sums one slice of the tile
// over distributed shared memory, in rank order, and writes it.  No
// partial leaves the chip, there is one launch per product, and the sum's
// order is fixed, so results are reproducible.
#pragma once

#include "common.cuh"

namespace qn {

// D += A B for one m16n8k16 bf16 tile (fp32 accumulate).  Not volatile: a
// pure function of its operands, so the compiler may schedule the operand
// loads of several MMAs ahead of them.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same MMA with a zero accumulator input: d = a b.
__device__ __forceinline__ void mma_bf16_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                 uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

constexpr int kSmallTile = 64;     // output rows per tile and reduction step length
constexpr int kMaxRank = 128;
constexpr int kMaxCluster = 8;
constexpr int kRankConsumerWarps = 8;   // two groups of 4, one 16-row block per warp of a group
constexpr int kRankConsumerThreads = kRankConsumerWarps * 32;
constexpr int kRankThreads = kRankConsumerThreads + 32;   // + 1 producer warp
constexpr int kRankIssuers = 4;        // producer lanes that issue copies
constexpr int kRankTileBytes = kSmallTile * 128;   // one 64 x 64 bf16 box, 128-byte swizzled
constexpr int kRankMaxStages = 8;

// Shared memory of one rank-r CTA: the ring (the partial tile reuses it) and
// its barriers, plus the slack that aligns the ring to 1024 bytes.
inline size_t rank_smem_bytes(int stages, int wboxes) {
  return 1024 + static_cast<size_t>(stages) * kRankTileBytes * (1 + wboxes) + 16 * kRankMaxStages;
}

struct SmallProblem {
  int kind;
  const __nv_bfloat16* X;   // down: [rows, red] ; up: [red, rows]
  const __nv_bfloat16* W;   // down: W(j, k) ; up: V [red, r]
  int w_transposed;         // down only: 0 -> W[j*red + k], 1 -> W[k*r + j]
  int64_t rows;             // output rows (M for down, P for up)
  int64_t red;              // reduction length (K for down, M for up)
  int64_t ldx, ldw;         // row strides (elements) of X and of the rank-side operand
  int r;
  int rj;                   // rank columns per tile (r / column splits)
  int csplit;               // column splits
  int64_t chunk;            // reduction elements per CTA of a cluster (multiple of 64)
  int tiles;                // ceil(rows / 64)
  float s;                  // output scale
  // down outputs
  __nv_bfloat16* plain;     // [rows, r] bf16(sum) with row stride ldp, or null
  __nv_bfloat16* scaled;    // [rows, rp] bf16(fl32(s * sum)) with `pad` zero columns after r, or null
  int64_t ldp;
  int rp, pad;
  // up output
  float* out;               // fl32(s * sum): [rows, r], or [r, rows] when transpose
  int transpose;
};

constexpr int kSmallMaxProblems = 4;

struct SmallBatch {
  SmallProblem p[kSmallMaxProblems];
  int count;
  int cend[kSmallMaxProblems];   // clusters of problems 0 .. i (tiles * csplit, summed)
  int clusters;             // clusters of all problems
  int cs;                   // CTAs per cluster (reduction splits)
  int wboxes;               // 64-column boxes of the rank-side operand per stage (1 or 2)
  int stages;               // ring depth, <= kRankMaxStages
};

// Tensor maps of the operands, all bf16 with 64 x 64 boxes and the 128-byte
// swizzle: x[i] is problem i's X, w[i] its rank-side operand (zero fill past
// rank r).
struct SmallMaps {
  CUtensorMap x[kSmallMaxProblems];
  CUtensorMap w[kSmallMaxProblems];
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// Byte offset of 16-byte chunk `c` of row `row` in a 128-byte-swizzled box
// (TMA stores chunk c of row r at chunk c ^ (r % 8); the box is 1024-aligned).
__device__ __forceinline__ uint32_t sw128(int row, int c) {
  return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
}

// Advances a ring position (slot, parity) by n steps.
__device__ __forceinline__ void ring_advance(int& stage, uint32_t& phase, int n, int stages) {
  const int t = stage + n;
  phase ^= static_cast<uint32_t>((t / stages) & 1);
  stage = t % stages;
}
// The same for 0 <= n <= stages, without a division (the loops' steps).
__device__ __forceinline__ void ring_step(int& stage, uint32_t& phase, int n, int stages) {
  stage += n;
  if (stage >= stages) {
    stage -= stages;
    phase ^= 1u;
  }
}

// One consumer warp's share of a tile's reduction steps for one operand
// layout: steps first, first + 2, ... (the two consumer groups take
// alternate steps; `stages` is even, so each group keeps to its own slots).
// The warp owns output rows 16 * wr .. + 15 and accumulates all of the
// tile's rank columns.  Layouts: 0 = down product with W stored [j][k];
// 1 = down product with W stored [k][j] (read transposed); 2 = up product
// (X and V both read transposed).  The ldmatrix row addresses of a lane
// within a stage are fixed, so they are computed once: in a 128-byte
// swizzled box, 16-byte chunk c of row y sits at y * 128 + ((c ^ (y % 8)) << 4),
// and every row a lane addresses has y % 8 == lane % 8.
template <int NT, int LAYOUT>
__device__ __forceinline__ void rank_steps(float (&acc)[NT][4], uint32_t ring, int stage_bytes, int stages,
                                           int stage, uint32_t phase, int nsteps, int first, uint64_t* full,
                                           uint64_t* empty, volatile int* abort_flag, int wr, int lane) {
  const int mi = lane >> 3, rr = lane & 7;
  constexpr int kPairs = (NT + 1) / 2;
  uint32_t offA[4], offB[4], colB[kPairs];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // A[m][k] = X[m][k]: matrices (m 0-7, k 0-7), (m 8-15, k 0-7), (m 0-7, k 8-15), (m 8-15, k 8-15)
    offA[i] = static_cast<uint32_t>((wr * 16 + (mi & 1) * 8 + rr) * 128 + (((2 * i + (mi >> 1)) ^ rr) << 4));
    // B[k][j] = W[j][k]: (j 0-7, k 0-7), (j 0-7, k 8-15), (j 8-15, k 0-7), (j 8-15, k 8-15), j = 8t + ..
    offB[i] = static_cast<uint32_t>(((mi >> 1) * 8 + rr) * 128 + (((2 * i + (mi & 1)) ^ rr) << 4));
  }
  // up product: A[p][m] = X[m][p] read transposed, rows m = 16i + (mi >> 1) * 8 + rr
  const uint32_t offAt = static_cast<uint32_t>(((mi >> 1) * 8 + rr) * 128 + (((2 * wr + (mi & 1)) ^ rr) << 4));
#pragma unroll
  for (int tp = 0; tp < kPairs; ++tp) {
    // B[k][j] stored k-major, read transposed: (k 0-7, j 0-7), (k 8-15, j 0-7), (k 0-7, j 8-15),
    // (k 8-15, j 8-15); rows k = 16i + (mi & 1) * 8 + rr, chunk c = 2tp + (mi >> 1) of 8 columns
    const int c = 2 * tp + (mi >> 1);
    colB[tp] = static_cast<uint32_t>(((mi & 1) * 8 + rr) * 128 + kRankTileBytes * (c >> 3) + (((c & 7) ^ rr) << 4));
  }
  ring_advance(stage, phase, first, stages);
  for (int step = first; step < nsteps; step += 2) {
    if (!mbar_wait(&full[stage], phase, abort_flag, ERR_RANK_WAIT)) break;
    const uint32_t sx = ring + static_cast<uint32_t>(stage * stage_bytes);
    const uint32_t sw = sx + kRankTileBytes;
    // the four 16-wide k-steps unrolled: their shared-memory loads overlap
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t a0, a1, a2, a3;
      if (LAYOUT == 2) ldsm_x4_t(sx + offAt + i * 2048, a0, a1, a2, a3);
      else ldsm_x4(sx + offA[i], a0, a1, a2, a3);
#pragma unroll
      for (int t = 0; t < NT; t += 2) {
        uint32_t b0, b1, b2, b3;
        if (LAYOUT == 0) ldsm_x4(sw + offB[i] + t * 1024, b0, b1, b2, b3);
        else ldsm_x4_t(sw + colB[t / 2] + i * 2048, b0, b1, b2, b3);
        mma_bf16_16816(acc[t], a0, a1, a2, a3, b0, b1);
        if (t + 1 < NT) mma_bf16_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    ring_step(stage, phase, 2, stages);
  }
}

// One tile (64 output rows x the tile's rj = 8 * NT rank columns) belongs
// to a cluster of batch.cs CTAs that split the reduction.  In each CTA, warp
// 8 streams 64-step boxes of X and of the rank-side operand into a ring with
// TMA (one elected thread issues, the warp keeps the ring position).  The
// eight consumer warps form two groups that take alternate stages; in each
// group, warp w owns output rows 16w .. 16w + 15 and runs ldmatrix + mma.sync
// on them.  A consumer warp's instruction stream is a chain of dependent
// shared-memory loads and MMAs, so two groups keep twice the work in flight.
// The groups' partial tiles are added (group 0's + group 1's), then the
// cluster's partial tiles are combined over distributed shared memory.
// CTAs loop over tiles when the grid has fewer clusters than tiles.
template <int NT>
__global__ void __launch_bounds__(kRankThreads) lora_rank_kernel(const __grid_constant__ SmallMaps maps,
                                                                 SmallBatch batch) {
  extern __shared__ uint8_t rank_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rank_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int stages = batch.stages;
  const int stage_bytes = kRankTileBytes * (1 + batch.wboxes);
  float* red = reinterpret_cast<float*>(smem);     // [64][rj], reuses the ring between tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + kRankMaxStages;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == kRankConsumerThreads) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    abort_flag = 0;
    fence_barrier_init();
    for (int i = 0; i < batch.count; ++i) {
      tma_prefetch_desc(&maps.x[i]);
      tma_prefetch_desc(&maps.w[i]);
    }
  }
  __syncthreads();
  // The inputs of this kernel may be written by the preceding kernel.  The
  // next kernel may start only after that wait: it reads inputs of the call
  // without waiting itself.
  pdl_wait_primary();
  pdl_launch_dependents();

  const int cs = batch.cs;
  const int q_rank = static_cast<int>(cluster_ctarank());
  const int g = lane >> 2, q = lane & 3;
  const int grp = warp >> 2, wr = warp & 3;      // consumer group, row block
  const uint32_t smem0 = smem_u32(smem);
  int stage = 0;                                 // ring position, the same in every role
  uint32_t phase = 0;

  for (int clg = blockIdx.x / cs; clg < batch.clusters; clg += gridDim.x / cs) {
    int pi = 0;
    while (pi + 1 < batch.count && clg >= batch.cend[pi]) ++pi;
    const int cl = pi ? clg - batch.cend[pi - 1] : clg;
    const SmallProblem P = batch.p[pi];            // by value: fields live in registers
    const int tile = cl % P.tiles;
    const int csp = cl / P.tiles;
    const int j0 = csp * P.rj;
    const int64_t row0 = static_cast<int64_t>(tile) * kSmallTile;
    const int64_t k_begin = static_cast<int64_t>(q_rank) * P.chunk;
    int64_t k_end = k_begin + P.chunk;
    if (k_end > P.red) k_end = P.red;
    const int nsteps = k_end > k_begin ? static_cast<int>((k_end - k_begin + kSmallTile - 1) / kSmallTile) : 0;
    const int r = P.r, rj = P.rj;
    const int kind = P.kind, wtr = P.w_transposed;

    if (warp == kRankConsumerWarps) {
      // ---------------------------------------------------------- producer
      // Lanes 0 .. P - 1, P = min(kRankIssuers, stages), each fill every P-th
      // stage.  On B200 the copies of one issuing thread complete about one
      // stage per memory round trip however deep the ring is, so a single
      // issuing thread capped a CTA at about 20 GB/s; the stream grows with
      // the issuing lanes.
      // A lane waits for its slot's previous use to be released; the wait is
      // on a parity, so it must not reach the slot two uses ahead: with no
      // more issuing lanes than stages, the use two laps back was released
      // before the lane issued its previous stage.
      const int issuers = stages < kRankIssuers ? stages : kRankIssuers;
      if (lane < issuers) {
        const CUtensorMap* mx = &maps.x[pi];
        const CUtensorMap* mw = &maps.w[pi];
        int st = stage;
        uint32_t ph = phase;
        ring_advance(st, ph, lane, stages);
        for (int step = lane; step < nsteps; step += issuers) {
          if (!mbar_wait(&empty[st], ph ^ 1, &abort_flag, ERR_RANK_WAIT)) break;
          uint8_t* sx = smem + st * stage_bytes;
          const int k0 = static_cast<int>(k_begin + static_cast<int64_t>(step) * kSmallTile);
          mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(stage_bytes));
          if (kind == 0) tma_load_2d(mx, &full[st], sx, k0, static_cast<int>(row0));
          else tma_load_2d(mx, &full[st], sx, static_cast<int>(row0), k0);
          for (int b = 0; b < batch.wboxes; ++b) {
            uint8_t* sw = sx + kRankTileBytes * (1 + b);
            if (kind == 0 && !wtr) tma_load_2d(mw, &full[st], sw, k0, j0 + 64 * b);
            else tma_load_2d(mw, &full[st], sw, j0 + 64 * b, k0);
          }
          ring_step(st, ph, issuers, stages);
        }
      }
      __syncwarp();
      ring_advance(stage, phase, nsteps, stages);
    } else {
      // ---------------------------------------------------------- consumers
      float acc[NT][4];
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
      if (kind == 1)
        rank_steps<NT, 2>(acc, smem0, stage_bytes, stages, stage, phase, nsteps, grp, full, empty, &abort_flag, wr, lane);
      else if (wtr)
        rank_steps<NT, 1>(acc, smem0, stage_bytes, stages, stage, phase, nsteps, grp, full, empty, &abort_flag, wr, lane);
      else
        rank_steps<NT, 0>(acc, smem0, stage_bytes, stages, stage, phase, nsteps, grp, full, empty, &abort_flag, wr, lane);
      ring_advance(stage, phase, nsteps, stages);
      // this CTA's partial tile, red[row][j] = group 0's + group 1's, over the
      // ring once every consumer warp is done reading it
      named_bar_sync(1, kRankConsumerThreads);
      const int ro = wr * 16 + g;
      if (grp == 1) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int j = 8 * t + 2 * q;
          *reinterpret_cast<float2*>(&red[ro * rj + j]) = make_float2(acc[t][0], acc[t][1]);
          *reinterpret_cast<float2*>(&red[(ro + 8) * rj + j]) = make_float2(acc[t][2], acc[t][3]);
        }
      }
      named_bar_sync(1, kRankConsumerThreads);
      if (grp == 0) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int j = 8 * t + 2 * q;
          float2* lo = reinterpret_cast<float2*>(&red[ro * rj + j]);
          float2* hi = reinterpret_cast<float2*>(&red[(ro + 8) * rj + j]);
          const float2 o0 = *lo, o1 = *hi;
          *lo = make_float2(acc[t][0] + o0.x, acc[t][1] + o0.y);
          *hi = make_float2(acc[t][2] + o1.x, acc[t][3] + o1.y);
        }
      }
      // the ring is refilled by TMA (async proxy) after these plain stores
      fence_proxy_async_smem();
    }
    cluster_sync_all();
    // Every CTA of the cluster reduces its own slice of the tile: groups of
    // four partial values are read from all cs CTAs first, then added in rank
    // order (a fixed order, so the result is reproducible).
    if (warp < kRankConsumerWarps) {
      const uint32_t red0 = smem_u32(red);
      const int nvec = kSmallTile * rj / 4;
      const int per = (nvec + cs - 1) / cs;
      const int v0 = q_rank * per;
      const int v1 = min(nvec, v0 + per);
      for (int v = v0 + tid; v < v1; v += kRankConsumerThreads) {
        float4 part[kMaxCluster];
#pragma unroll
        for (int c = 0; c < kMaxCluster; ++c)
          if (c < cs) part[c] = ld_cluster_f32x4(map_to_rank(red0 + 16u * v, c));
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
        if (kind == 0) {
          if (P.plain) {
#pragma unroll
            for (int u = 0; u < 4; ++u) P.plain[row * P.ldp + jj + u] = __float2bfloat16_rn(e[u]);
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
      if (kind == 0 && P.scaled && csp == 0 && q_rank == 0 && P.pad > 0) {
        const int pad = P.pad;
        for (int i = tid; i < kSmallTile * pad; i += kRankConsumerThreads) {
          const int64_t row = row0 + i / pad;
          if (row < P.rows) P.scaled[row * P.rp + r + i % pad] = __float2bfloat16_rn(0.f);
        }
      }
    }
    // Keep every CTA's partial tile alive until all CTAs have read it; only
    // then may the next tile's copies overwrite the ring.
    cluster_sync_all();
  }
}

}  // namespace qn
