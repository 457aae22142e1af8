// gemv.cuh -- decode-shape forward (1..16 tokens): the NF4 GEMV.
//
// [QLoRA glossary, "Come funziona QLoRA": the frozen layer dequantizes its
//  NF4 weights just before the matmul and adds the LoRA path's output.]
//
// y[t][n] = sum_b s_hat(n, b) * sum_{k in block b} x[t][k] * level[code(n, k)]
//         + sum_j us[t][j] * B[n][j]               (us = bf16(s * x A^T))
//
// HBM-bound: each packed code byte is read once, straight into registers.
// Work layout:
//  * a CTA owns a contiguous range of 8-row groups of W and all of K; its
//    work is cut into units of one 8-row group x one k-range of 256 (four
//    64-weight blocks), numbered k-range-major, and each warp takes a
//    contiguous run of units, so that its x fragments change only when its
//    k-range does;
//  * no barrier and no wait in the main loop: every warp keeps kDepth units'
//    code loads (four 8-byte loads per thread per unit) and scale inputs in
//    flight in registers ahead of the unit it computes;
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
//  * the block scale multiplies the block's fp32 partial product (the scale
//    is constant over the block), so the tensor core sees the levels;
//  * each unit's 16 x 8 partial tile is parked in shared memory; at the end
//    the tiles of a row group are summed over k-ranges in k order, the LoRA
//    product is added (after the kernel that computes us, which this one may
//    overlap, has finished) and y is written.
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
constexpr int kGemvDepth = 3;                       // units in flight per warp ahead of the one computed

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

// Streaming 8-byte load that does not allocate in L1.
__device__ __forceinline__ uint2 ldg_stream_u2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// The table word of code byte k (0..3) of `w` for this lane: lane4 holds
// lane * 4 in its low byte, and one byte permute puts byte k of w above it.
__device__ __forceinline__ uint32_t gemv_lookup(uint32_t tbl, uint32_t w, uint32_t lane4, int k) {
  const uint32_t off = __byte_perm(w, lane4, 0x7604u | (static_cast<uint32_t>(k) << 4));
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(tbl + off));
  return v;
}

// One unit's loads.  NF4: this thread's 8 code bytes of each of the 4
// blocks of its weight row, and the scale inputs of (row, block q).  bf16
// weights: the 16 weights of each block that the codes would stand for
// (columns 64 b + 16 q .. + 15), 8 words per block.
template <bool kBF16W>
struct GemvUnitIn {
  uint2 c[4];
  int q8;
  float step, mean;
};
template <>
struct GemvUnitIn<true> {
  uint4 a[4][2];
};

template <bool kBF16W>
__device__ __forceinline__ void gemv_load_unit(const GemvParams& p, int64_t row, int kr, int q, GemvUnitIn<kBF16W>& u) {
  if constexpr (kBF16W) {
    const uint4* src = reinterpret_cast<const uint4*>(p.wb + row * p.K + static_cast<int64_t>(kr) * 256 + 16 * q);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      u.a[b][0] = __ldg(src + 8 * b);
      u.a[b][1] = __ldg(src + 8 * b + 1);
    }
  } else {
    const uint8_t* src = p.codes + row * (p.K >> 1) + static_cast<int64_t>(kr) * 128 + 8 * q;
#pragma unroll
    for (int b = 0; b < 4; ++b) u.c[b] = ldg_stream_u2(src + 32 * b);
    const int64_t si = row * p.kb + static_cast<int64_t>(kr) * 4 + q;
    u.q8 = __ldg(p.qscale + si);
    u.step = __ldg(p.dq_step + (si >> 8));
    u.mean = __ldg(p.dq_mean + (si >> 8));
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

template <int NH, bool kBF16W = false>
__global__ void __launch_bounds__(GemvCfg<NH>::kThreads, 1) qlora_gemv_kernel(GemvParams p) {
  constexpr int W = GemvCfg<NH>::kWarps;
  constexpr int D = kBF16W ? 1 : kGemvDepth;
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  float* red = reinterpret_cast<float*>(gemv_smem + kGemvTableBytes);   // [unit][8 rows][T]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const uint32_t tbl = smem_u32(gemv_smem);
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;

  pdl_launch_dependents();

  // byte -> (bf16(level[lo]), bf16(level[hi])), one copy per lane
  if constexpr (!kBF16W) {
    for (int i = tid; i < 256 * 32; i += W * 32) {
      const int e = i >> 5;
      reinterpret_cast<uint32_t*>(gemv_smem)[e * 64 + (i & 31)] = pack_bf16x2(p.lv.v[e & 15], p.lv.v[e >> 4]);
    }
  }

  const int rg_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.nrg / gridDim.x);
  const int rg_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.nrg / gridDim.x);
  const int T = p.T;

  for (int rb0 = rg_begin; rb0 < rg_end; rb0 += p.rg_batch) {
    const int nrb = min(p.rg_batch, rg_end - rb0);
    const int units = p.nkr * nrb;
    const int i0 = static_cast<int>(static_cast<int64_t>(warp) * units / W);
    const int i1 = static_cast<int>(static_cast<int64_t>(warp + 1) * units / W);
    __syncthreads();      // the table is built; the previous batch's tiles are consumed

    GemvUnitIn<kBF16W> in[D];
    // (k-range, row group) of the unit computed next and of the unit loaded
    // next, stepped without divisions
    int kr_c = i0 / max(nrb, 1), rg_c = i0 - kr_c * nrb;
    int kr_p = kr_c, rg_p = rg_c;
#pragma unroll
    for (int j = 0; j < D; ++j)
      if (i0 + j < i1) {
        gemv_load_unit(p, static_cast<int64_t>(rb0 + rg_p) * 8 + g, kr_p, q, in[j]);
        if (++rg_p == nrb) { rg_p = 0; ++kr_p; }
      }
    uint32_t xf[NH][4][8];
    int cur_kr = -1;

    for (int ib = i0; ib < i1; ib += D) {
#pragma unroll
      for (int j = 0; j < D; ++j) {
        const int i = ib + j;
        if (i < i1) {
          const int kr = kr_c, rgl = rg_c;
          if (++rg_c == nrb) { rg_c = 0; ++kr_c; }
          if (kr != cur_kr) {
            gemv_load_x<NH>(p, kr, g, q, xf);
            cur_kr = kr;
          }
          const GemvUnitIn<kBF16W> u = in[j];
          if (i + D < i1) {
            gemv_load_unit(p, static_cast<int64_t>(rb0 + rg_p) * 8 + g, kr_p, q, in[j]);
            if (++rg_p == nrb) { rg_p = 0; ++kr_p; }
          }
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          if constexpr (kBF16W) {
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
          } else {
            // scale of (row g, block q); rows 2q and 2q+1 of block b come from lanes 8q + b and 8q + 4 + b
            const float sh = restore_scale(static_cast<int8_t>(u.q8), u.step, u.mean);
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const float s0 = __shfl_sync(0xFFFFFFFFu, sh, 8 * q + b);
              const float s1 = __shfl_sync(0xFFFFFFFFu, sh, 8 * q + 4 + b);
              float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                const uint32_t w = (m < 2) ? u.c[b].x : u.c[b].y;
                const uint32_t b0 = gemv_lookup(tbl, w, lane4, 2 * (m & 1));
                const uint32_t b1 = gemv_lookup(tbl, w, lane4, 2 * (m & 1) + 1);
                const uint32_t a0 = xf[0][b][2 * m], a2 = xf[0][b][2 * m + 1];
                const uint32_t a1 = NH == 2 ? xf[NH - 1][b][2 * m] : 0u;
                const uint32_t a3 = NH == 2 ? xf[NH - 1][b][2 * m + 1] : 0u;
                mma_bf16_16816(t, a0, a1, a2, a3, b0, b1);
              }
              acc[0] = fmaf(s0, t[0], acc[0]);
              acc[1] = fmaf(s1, t[1], acc[1]);
              acc[2] = fmaf(s0, t[2], acc[2]);
              acc[3] = fmaf(s1, t[3], acc[3]);
            }
          }
          // this unit's tile: rows 2q, 2q+1 for tokens g and g+8
          float* rt = red + static_cast<int64_t>(kr * nrb + rgl) * 8 * T;
          if (g < T) {
            rt[(2 * q) * T + g] = acc[0];
            rt[(2 * q + 1) * T + g] = acc[1];
          }
          if (g + 8 < T) {
            rt[(2 * q) * T + g + 8] = acc[2];
            rt[(2 * q + 1) * T + g + 8] = acc[3];
          }
        }
      }
    }
    __syncthreads();
    if (!kBF16W && p.wait_us) pdl_wait_primary();
    // y[t][n] for the batch's rows: the k-range tiles in k order, + LoRA
    const int outs = nrb * 8 * T;
    for (int o = tid; o < outs; o += W * 32) {
      const int t = o / (nrb * 8);
      const int nl = o - t * (nrb * 8);          // row within the batch (fastest: coalesced y)
      const int rgl = nl >> 3, row = nl & 7;
      float sum = 0.f;
      for (int kr = 0; kr < p.nkr; ++kr) sum += red[(static_cast<int64_t>(kr * nrb + rgl) * 8 + row) * T + t];
      const int64_t n = static_cast<int64_t>(rb0) * 8 + nl;
      if constexpr (kBF16W) {
        const __nv_bfloat16 ub = __float2bfloat16_rn(sum);
        if (p.u_out) p.u_out[static_cast<int64_t>(t) * p.N + n] = ub;
        p.us_out[static_cast<int64_t>(t) * p.us_ld + n] = __float2bfloat16_rn(__fmul_rn(p.s, sum));
        continue;
      }
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

}  // namespace qn
