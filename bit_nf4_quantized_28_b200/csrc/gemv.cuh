// gemv.cuh -- decode-shape forward (1..16 tokens): the NF4 GEMV.
//
// [QLoRA glossary, "Come funziona QLoRA": the frozen layer dequantizes its
//  NF4 weights just before the matmul and adds the LoRA path's output.]
//
// y[t][n] = sum_b s_hat(n, b) * sum_{k in block b} x[t][k] * level[code(n, k)]
//         + sum_j us[t][j] * B[n][j]               (us = bf16(s * x A^T))
//
// HBM-bound: each packed code byte is read once.  Work layout:
//  * a CTA owns a contiguous range of 8-row groups of W and all of K; its
//    work is cut into units of one 8-row group x one k-range of 256 (four
//    64-weight blocks), numbered k-range-major, and each warp takes a
//    contiguous run of units, so that its x fragments change only when its
//    k-range does;
//  * every warp streams its units' codes through its own ring of shared-
//    memory stages: lane 0 requests each unit (8 rows x 128 bytes, one TMA
//    box) several units ahead, and the warp waits on that stage's barrier;
//    no barrier couples the warps in the main loop;
//  * the block scales of the CTA's rows are restored once (per batch of row
//    groups) into shared memory; the block scale multiplies the block's fp32
//    partial product (it is constant over the block), so the tensor core sees
//    the levels;
//  * mma.sync m16n8k16 with the tokens as the 16-row A operand (x, in
//    registers) and 8 weight rows as the B operand; inside a block the k order
//    of an MMA is permuted so that a thread's B values come from 8 consecutive
//    code bytes of its weight row and its x values from 16 consecutive
//    columns; both operands use the same permutation, so the sum is unchanged;
//  * a code byte becomes a bf16 pair (level[low nibble], level[high nibble])
//    through a 256-entry table stored once per lane: entry e of lane l sits at
//    byte e * 256 + l * 4 (no bank conflicts), so one byte permute that puts
//    the code byte in bits 8..15 and the lane's offset in bits 0..7 forms the
//    address;
//  * each unit's 16 x 8 partial tile is parked in shared memory; at the end
//    of a batch the tiles of a row group are summed over k-ranges in k order,
//    the LoRA product is added (after the kernel that computes us, which this
//    one may overlap, has finished) and y is written.
// u = x A^T runs through the same unit layout on bf16 weights
// (lora_down_gemv_kernel), on a few CTAs beside the NF4 GEMV.
#pragma once

#include "common.cuh"
#include "lora_small.cuh"
#include "nf4_storage.cuh"

namespace qn {

struct GemvParams {
  const uint8_t* codes;       // [N, K/2]
  const int8_t* qscale;       // [N*K/64]
  const float* dq_step;
  const float* dq_mean;
  const __nv_bfloat16* x;     // [T, K]
  int T;
  int64_t N, K;
  int kb;                     // K / 64
  int nkr;                    // K / 256 (k-ranges)
  int nrg;                    // N / 8 (row groups)
  int rg_batch;               // row groups whose partial tiles shared memory holds at once
  int wait_us;                // wait for the preceding kernel (it writes us) before the final step
  int wait_all;               // wait for the preceding kernel before reading any input
  const __nv_bfloat16* B;     // [N, r], or null without LoRA
  const __nv_bfloat16* us;    // [T, rp] = bf16(s * x A^T)
  int r, rp;
  __nv_bfloat16* y;           // [T, N]
  // bf16-weight mode (u = x A^T): the weight is wb [N, K] (N = r) and the
  // outputs are u [T, N] (u_out, when given) and bf16(s u) [T, us_ld]
  const __nv_bfloat16* wb;
  float s;
  __nv_bfloat16* u_out;
  __nv_bfloat16* us_out;
  int us_ld;
  Levels lv;
};

constexpr int kGemvTableBytes = 256 * 256;
constexpr int kGemvSmemBudget = 227 * 1024 - 1024;   // dynamic bytes
constexpr int kGemvRing = 4;                        // code stages per warp (units requested ahead)
constexpr int kGemvStageBytes = 1024;               // one unit's codes: 8 rows x 128 bytes

// NH = 1: up to 8 tokens; NH = 2: up to 16.
template <int NH>
struct GemvCfg {
  static constexpr int kWarps = NH == 1 ? 16 : 12;
  static constexpr int kThreads = kWarps * 32;
};

// Bytes of partial tiles for `rgs` row groups of all k-ranges.
__host__ __device__ constexpr int64_t gemv_red_bytes(int nkr, int rgs, int T) {
  return static_cast<int64_t>(nkr) * rgs * 8 * T * 4;
}

// The table word of code byte k (0..3) of `w` for this lane: lane4 holds
// lane * 4 in its low byte, and one byte permute puts byte k of w above it.
// A plain load, so the compiler can issue many ahead of the MMAs that use them.
__device__ __forceinline__ uint32_t gemv_lookup(const uint8_t* tbl, uint32_t w, uint32_t lane4, int k) {
  const uint32_t off = __byte_perm(w, lane4, 0x7604u | (static_cast<uint32_t>(k) << 4));
  return *reinterpret_cast<const uint32_t*>(tbl + off);
}

// One unit of bf16 weights (u = x A^T): the 16 weights of each of its 4
// blocks that this thread multiplies (columns 64 b + 16 q .. + 15 of row g).
struct GemvBf16Unit {
  uint4 a[4][2];
};

__device__ __forceinline__ void gemv_load_bf16_unit(const GemvParams& p, int64_t row, int kr, int q, GemvBf16Unit& u) {
  const uint4* src = reinterpret_cast<const uint4*>(p.wb + row * p.K + static_cast<int64_t>(kr) * 256 + 16 * q);
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    u.a[b][0] = __ldg(src + 8 * b);
    u.a[b][1] = __ldg(src + 8 * b + 1);
  }
}

// x fragments of one k-range for tokens g (and g + 8): per block b, the 16
// consecutive columns 64 b + 16 q .. + 15 (8 words).
template <int NH>
__device__ __forceinline__ void gemv_load_x(const GemvParams& p, int kr, int g, int q, uint32_t (&xf)[NH][4][8]) {
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const int tok = g + 8 * h;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
      if (tok < p.T) {
        const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(tok) * p.K +
                                                          static_cast<int64_t>(kr) * 256 + 64 * b + 16 * q);
        v0 = __ldg(src);
        v1 = __ldg(src + 1);
      }
      xf[h][b][0] = v0.x; xf[h][b][1] = v0.y; xf[h][b][2] = v0.z; xf[h][b][3] = v0.w;
      xf[h][b][4] = v1.x; xf[h][b][5] = v1.y; xf[h][b][6] = v1.z; xf[h][b][7] = v1.w;
    }
  }
}

// Sums a batch's parked tiles over the k-ranges in k order and writes the
// outputs: the NF4 layer's y (+ the LoRA product), or u and bf16(s u).
template <bool kBF16W>
__device__ __forceinline__ void gemv_finish(const GemvParams& p, const float* red, int rb0, int nrb, int nthreads) {
  const int T = p.T;
  const int outs = nrb * 8 * T;
  for (int o = threadIdx.x; o < outs; o += nthreads) {
    const int t = o / (nrb * 8);
    const int nl = o - t * (nrb * 8);          // row within the batch (fastest: coalesced y)
    const int rgl = nl >> 3, row = nl & 7;
    float sum = 0.f;
    for (int kr = 0; kr < p.nkr; ++kr) sum += red[(static_cast<int64_t>(kr * nrb + rgl) * 8 + row) * T + t];
    const int64_t n = static_cast<int64_t>(rb0) * 8 + nl;
    if constexpr (kBF16W) {
      if (p.u_out) p.u_out[static_cast<int64_t>(t) * p.N + n] = __float2bfloat16_rn(sum);
      p.us_out[static_cast<int64_t>(t) * p.us_ld + n] = __float2bfloat16_rn(__fmul_rn(p.s, sum));
    } else {
      if (p.B) {
        const uint4* b8 = reinterpret_cast<const uint4*>(p.B + n * p.r);
        const uint4* u8 = reinterpret_cast<const uint4*>(p.us + static_cast<int64_t>(t) * p.rp);
        float lora = 0.f;
        for (int c = 0; c < p.r / 8; ++c) {
          const uint4 bv = __ldg(b8 + c), uv = u8[c];
          const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            lora = fmaf(__uint_as_float(uw[e] << 16), __uint_as_float(bw[e] << 16), lora);
            lora = fmaf(__uint_as_float(uw[e] & 0xFFFF0000u), __uint_as_float(bw[e] & 0xFFFF0000u), lora);
          }
        }
        sum += lora;
      }
      p.y[static_cast<int64_t>(t) * p.N + n] = __float2bfloat16_rn(sum);
    }
  }
}

// Parks a unit's 16 x 8 tile (rows 2q, 2q+1 for tokens g and g + 8).
__device__ __forceinline__ void gemv_park(float* red, int slot, int T, int g, int q, const float (&acc)[4]) {
  float* rt = red + static_cast<int64_t>(slot) * 8 * T;
  if (g < T) {
    rt[(2 * q) * T + g] = acc[0];
    rt[(2 * q + 1) * T + g] = acc[1];
  }
  if (g + 8 < T) {
    rt[(2 * q) * T + g + 8] = acc[2];
    rt[(2 * q + 1) * T + g + 8] = acc[3];
  }
}

// Shared memory of the NF4 GEMV: the lookup table, the warps' code rings,
// their barriers, the batch's restored block scales and its parked tiles.
struct GemvSmem {
  uint32_t ring, bars, scales, red, total;
};
__host__ __device__ constexpr GemvSmem gemv_smem_layout(int warps, int nkr, int rg_batch, int T, int kb) {
  GemvSmem L{};
  L.ring = kGemvTableBytes;
  L.bars = L.ring + static_cast<uint32_t>(warps) * kGemvRing * kGemvStageBytes;
  L.scales = L.bars + static_cast<uint32_t>(warps) * kGemvRing * 8;
  L.red = L.scales + static_cast<uint32_t>(rg_batch) * 8 * kb * 4;
  L.total = L.red + static_cast<uint32_t>(gemv_red_bytes(nkr, rg_batch, T));
  return L;
}

// The NF4 GEMV.  Each warp streams its units' codes through a ring of
// kGemvRing shared-memory stages: lane 0 requests a unit's 8 rows x 128
// bytes as one TMA box (128-byte swizzle) kGemvRing units ahead, and the
// warp waits for it on the stage's barrier (bounded).  The block scales of
// the CTA's rows are restored once per batch into shared memory.
template <int NH>
__global__ void __launch_bounds__(GemvCfg<NH>::kThreads, 1)
    qlora_gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, GemvParams p) {
  constexpr int W = GemvCfg<NH>::kWarps;
  constexpr int D = kGemvRing;
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  __shared__ int abort_flag;
  const GemvSmem L = gemv_smem_layout(W, p.nkr, p.rg_batch, p.T, p.kb);
  float* red = reinterpret_cast<float*>(gemv_smem + L.red);
  float* stab = reinterpret_cast<float*>(gemv_smem + L.scales);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const uint8_t* tbl = gemv_smem;
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
  uint8_t* ring = gemv_smem + L.ring + static_cast<uint32_t>(warp) * D * kGemvStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(gemv_smem + L.bars) + warp * D;

  if (lane == 0) {
    for (int j = 0; j < D; ++j) mbar_init(&full[j], 1);
    fence_barrier_init();
    if (warp == 0) tma_prefetch_desc(&tm_codes);
  }
  if (tid == 0) abort_flag = 0;
  pdl_launch_dependents();

  // byte -> (bf16(level[lo]), bf16(level[hi])), one copy per lane
  for (int i = tid; i < 256 * 32; i += W * 32) {
    const int e = i >> 5;
    reinterpret_cast<uint32_t*>(gemv_smem)[e * 64 + (i & 31)] = pack_bf16x2(p.lv.v[e & 15], p.lv.v[e >> 4]);
  }
  // as the first kernel of a call (launched to overlap the previous kernel's
  // tail), wait for the preceding work before reading any input
  if (p.wait_all) pdl_wait_primary();

  const int rg_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.nrg / gridDim.x);
  const int rg_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.nrg / gridDim.x);
  const int T = p.T;
  int uses = 0;          // ring uses of this warp so far (stage = uses % D)
  bool ok = true;

  for (int rb0 = rg_begin; rb0 < rg_end && ok; rb0 += p.rg_batch) {
    const int nrb = min(p.rg_batch, rg_end - rb0);
    const int units = p.nkr * nrb;
    const int i0 = static_cast<int>(static_cast<int64_t>(warp) * units / W);
    const int i1 = static_cast<int>(static_cast<int64_t>(warp + 1) * units / W);
    __syncthreads();      // barriers set up; the previous batch's scales and tiles are consumed

    // the warp's first units: request them before anything else
    int kr_p = i0 / max(nrb, 1), rg_p = i0 - kr_p * nrb;
    if (lane == 0) {
      for (int j = 0; j < D && i0 + j < i1; ++j) {
        uint64_t* bar = &full[(uses + j) % D];
        mbar_arrive_expect_tx(bar, kGemvStageBytes);
        tma_load_2d(&tm_codes, bar, ring + ((uses + j) % D) * kGemvStageBytes, kr_p * 128, (rb0 + rg_p) * 8);
        if (++rg_p == nrb) { rg_p = 0; ++kr_p; }
      }
    }
    kr_p = __shfl_sync(0xFFFFFFFFu, kr_p, 0);
    rg_p = __shfl_sync(0xFFFFFFFFu, rg_p, 0);

    // the batch's block scales s_hat, [row][block]: 16 consecutive scale
    // codes per thread (one 16-byte load; they share one group of 256), all
    // loads issued before any is used
    {
      const int n16 = nrb * 8 * p.kb / 16;
      const int64_t base = static_cast<int64_t>(rb0) * 8 * p.kb;
      for (int v0 = tid; v0 < n16; v0 += 2 * W * 32) {
        int4 qv[2];
        float st[2], mn[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int v = v0 + h * W * 32;
          if (v < n16) {
            const int64_t si = base + 16 * static_cast<int64_t>(v);
            qv[h] = __ldg(reinterpret_cast<const int4*>(p.qscale + si));
            st[h] = __ldg(p.dq_step + (si >> 8));
            mn[h] = __ldg(p.dq_mean + (si >> 8));
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int v = v0 + h * W * 32;
          if (v < n16) {
            const uint32_t words[4] = {static_cast<uint32_t>(qv[h].x), static_cast<uint32_t>(qv[h].y),
                                       static_cast<uint32_t>(qv[h].z), static_cast<uint32_t>(qv[h].w)};
            float4* dst = reinterpret_cast<float4*>(stab + 16 * v);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float f[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                f[e] = restore_scale(static_cast<int8_t>((words[c] >> (8 * e)) & 0xFFu), st[h], mn[h]);
              dst[c] = make_float4(f[0], f[1], f[2], f[3]);
            }
          }
        }
      }
    }
    // x of the warp's first k-range, while the scales are being written
    uint32_t xf[NH][4][8];
    int cur_kr = -1;
    if (i0 < i1) {
      cur_kr = i0 / max(nrb, 1);
      gemv_load_x<NH>(p, cur_kr, g, q, xf);
    }
    __syncthreads();      // the table (first batch) and the scales are written

    int kr_c = i0 / max(nrb, 1), rg_c = i0 - kr_c * nrb;
    for (int i = i0; i < i1; ++i) {
      const int kr = kr_c, rgl = rg_c;
      if (++rg_c == nrb) { rg_c = 0; ++kr_c; }
      if (kr != cur_kr) {
        gemv_load_x<NH>(p, kr, g, q, xf);
        cur_kr = kr;
      }
      const int stage = uses % D;
      if (!mbar_wait(&full[stage], (uses / D) & 1, &abort_flag, ERR_GEMV_WAIT)) { ok = false; break; }
      const uint8_t* cb = ring + stage * kGemvStageBytes + g * 128;
      uint2 c[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int chunk = 2 * b + (q >> 1);
        c[b] = *reinterpret_cast<const uint2*>(cb + ((chunk ^ g) << 4) + 8 * (q & 1));
      }
      // the stage is refilled (async proxy) with the unit D ahead once every lane has read it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && i + D < i1) {
        mbar_arrive_expect_tx(&full[stage], kGemvStageBytes);
        tma_load_2d(&tm_codes, &full[stage], ring + stage * kGemvStageBytes, kr_p * 128, (rb0 + rg_p) * 8);
      }
      if (i + D < i1) {
        if (++rg_p == nrb) { rg_p = 0; ++kr_p; }
      }
      ++uses;
      // scales of rows 2q and 2q + 1 for the unit's 4 blocks
      const float4 sa = *reinterpret_cast<const float4*>(stab + (rgl * 8 + 2 * q) * p.kb + kr * 4);
      const float4 sb = *reinterpret_cast<const float4*>(stab + (rgl * 8 + 2 * q + 1) * p.kb + kr * 4);
      const float s0[4] = {sa.x, sa.y, sa.z, sa.w}, s1[4] = {sb.x, sb.y, sb.z, sb.w};
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t w = (m < 2) ? c[b].x : c[b].y;
          const uint32_t b0 = gemv_lookup(tbl, w, lane4, 2 * (m & 1));
          const uint32_t b1 = gemv_lookup(tbl, w, lane4, 2 * (m & 1) + 1);
          const uint32_t a1 = NH == 2 ? xf[NH - 1][b][2 * m] : 0u;
          const uint32_t a3 = NH == 2 ? xf[NH - 1][b][2 * m + 1] : 0u;
          mma_bf16_16816(t, xf[0][b][2 * m], a1, xf[0][b][2 * m + 1], a3, b0, b1);
        }
        acc[0] = fmaf(s0[b], t[0], acc[0]);
        acc[1] = fmaf(s1[b], t[1], acc[1]);
        acc[2] = fmaf(s0[b], t[2], acc[2]);
        acc[3] = fmaf(s1[b], t[3], acc[3]);
      }
      gemv_park(red, kr * nrb + rgl, T, g, q, acc);
    }
    __syncthreads();
    if (!ok || abort_flag) {
      ok = false;
      break;
    }
    if (p.wait_us) pdl_wait_primary();
    gemv_finish<false>(p, red, rb0, nrb, W * 32);
  }
  // after a wait gave up: let this warp's requested copies land before exit
  if (!ok && lane == 0) {
    volatile int dummy = 0;
    for (int j = 0; j < D; ++j) mbar_wait(&full[(uses + j) % D], ((uses + j) / D) & 1, &dummy, ERR_GEMV_WAIT);
  }
}

// u = x A^T for the decode path: the same unit layout on bf16 weights, each
// thread's 16 weights of a block straight from global memory into registers
// (a small product: one CTA per 8 rank rows).
template <int NH>
__global__ void __launch_bounds__(GemvCfg<NH>::kThreads, 1) lora_down_gemv_kernel(GemvParams p) {
  constexpr int W = GemvCfg<NH>::kWarps;
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  float* red = reinterpret_cast<float*>(gemv_smem);   // [unit][8 rows][T]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  pdl_launch_dependents();
  const int rg_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.nrg / gridDim.x);
  const int rg_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.nrg / gridDim.x);
  for (int rb0 = rg_begin; rb0 < rg_end; rb0 += p.rg_batch) {
    const int nrb = min(p.rg_batch, rg_end - rb0);
    const int units = p.nkr * nrb;
    const int i0 = static_cast<int>(static_cast<int64_t>(warp) * units / W);
    const int i1 = static_cast<int>(static_cast<int64_t>(warp + 1) * units / W);
    __syncthreads();
    uint32_t xf[NH][4][8];
    int cur_kr = -1;
    for (int i = i0; i < i1; ++i) {
      const int kr = i / nrb, rgl = i - kr * nrb;
      if (kr != cur_kr) {
        gemv_load_x<NH>(p, kr, g, q, xf);
        cur_kr = kr;
      }
      GemvBf16Unit u;
      gemv_load_bf16_unit(p, static_cast<int64_t>(rb0 + rgl) * 8 + g, kr, q, u);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t wv[8] = {u.a[b][0].x, u.a[b][0].y, u.a[b][0].z, u.a[b][0].w,
                                u.a[b][1].x, u.a[b][1].y, u.a[b][1].z, u.a[b][1].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t a1 = NH == 2 ? xf[NH - 1][b][2 * m] : 0u;
          const uint32_t a3 = NH == 2 ? xf[NH - 1][b][2 * m + 1] : 0u;
          mma_bf16_16816(acc, xf[0][b][2 * m], a1, xf[0][b][2 * m + 1], a3, wv[2 * m], wv[2 * m + 1]);
        }
      }
      gemv_park(red, kr * nrb + rgl, p.T, g, q, acc);
    }
    __syncthreads();
    gemv_finish<true>(p, red, rb0, nrb, W * 32);
  }
}

}  // namespace qn
