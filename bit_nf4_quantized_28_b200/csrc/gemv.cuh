// gemv.cuh -- decode-shape forward (1..16 tokens): split-K NF4 GEMV.
//
// [QLoRA glossary, "Come funziona QLoRA": the frozen layer dequantizes its
//  NF4 weights just before the matmul and adds the LoRA path's output.]
//
// y[t][n] = sum_b s_hat(n, b) * sum_{k in block b} x[t][k] * level[code(n, k)]
//         + sum_j us[t][j] * B[n][j]               (us = bf16(s * x A^T))
//
// HBM-bound: each packed code byte is read once.  Layout of the work:
//  * mma.sync m16n8k16 with 16 weight rows as the A operand and the tokens
//    as the 8-column B operand (two column halves for 9..16 tokens);
//  * inside each 64-weight block the k order of an MMA is permuted so that a
//    thread's A values come from 8 consecutive code bytes of its row (one
//    64-bit load) and its x values from 16 consecutive columns; both operands
//    use the same permutation, so the sum is unchanged;
//  * a code byte becomes a bf16 pair (level[low nibble], level[high nibble])
//    through a 256-entry table stored once per lane (conflict-free loads);
//  * the block scale multiplies the block's fp32 partial product (the scale
//    is constant over the block), so the tensor core sees the levels;
//  * warps 0..7 each keep the x fragments of a fixed range of blocks in
//    registers and loop over groups of 16 weight rows, prefetching the next
//    group's codes; warp 8 computes the LoRA product for the same rows;
//    the 9 partial tiles are summed through shared memory in a fixed order.
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
  const __nv_bfloat16* us;    // [T, rp] = bf16(s * x A^T), zero padded; null if no LoRA
  const __nv_bfloat16* B;     // [N, r]; null if no LoRA
  int T;
  int64_t N, K;
  int r, rp;
  int kb;                     // K / 64
  int split_blocks;           // weight blocks per k-split
  int ks;                     // k-splits
  int pcta;                   // persistent CTAs per k-split
  __nv_bfloat16* y;           // [T, N] when ks == 1
  float* partial;             // [ks, T, N] when ks > 1
  Levels lv;
};

constexpr int kGemvWeightWarps = 8;
constexpr int kGemvWarps = kGemvWeightWarps + 1;   // + the LoRA warp
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvMaxLoraBlocks = 2;               // r <= 128
constexpr size_t kGemvSmemBytes = 256 * 32 * 4 + 2 * kGemvWarps * 256 * 4;

template <int NH>
__device__ __forceinline__ void gemv_load_x(const __nv_bfloat16* base, int64_t ld, int T, int g,
                                            int q, int col0, bool valid, uint32_t (&f)[NH][8]) {
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const int tok = g + 8 * h;
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    if (valid && tok < T) {
      const __nv_bfloat16* src = base + static_cast<int64_t>(tok) * ld + col0 + 16 * q;
      v0 = *reinterpret_cast<const uint4*>(src);
      v1 = *reinterpret_cast<const uint4*>(src + 8);
    }
    f[h][0] = v0.x; f[h][1] = v0.y; f[h][2] = v0.z; f[h][3] = v0.w;
    f[h][4] = v1.x; f[h][5] = v1.y; f[h][6] = v1.z; f[h][7] = v1.w;
  }
}

template <int NH, int BPW>
__global__ void __launch_bounds__(kGemvThreads, 1) qlora_gemv_kernel(GemvParams p) {
  extern __shared__ __align__(16) uint8_t gemv_smem[];
  uint32_t* tbl = reinterpret_cast<uint32_t*>(gemv_smem);                 // [256][32]
  float* red = reinterpret_cast<float*>(gemv_smem + 256 * 32 * 4);        // [2][9][16][16]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;

  // byte -> (bf16(level[lo]), bf16(level[hi])), one copy per lane.
  for (int i = tid; i < 256 * 32; i += kGemvThreads) {
    const int b = i >> 5;
    tbl[i] = pack_bf16x2(p.lv.v[b & 15], p.lv.v[b >> 4]);
  }
  pdl_launch_dependents();
  pdl_wait_primary();
  __syncthreads();

  const int split = blockIdx.x / p.pcta;
  const int pidx = blockIdx.x % p.pcta;
  const int ngroups = static_cast<int>(p.N >> 4);
  const int64_t row_bytes = p.K >> 1;
  const uint32_t tbl_lane = smem_u32(tbl) + (lane << 2);
  const unsigned full = 0xFFFFFFFFu;

  int buf = 0;
  if (warp < kGemvWeightWarps) {
    // ---------------------------------------------------------- weight warps
    const int sb0 = split * p.split_blocks;
    int sb1 = sb0 + p.split_blocks;
    if (sb1 > p.kb) sb1 = p.kb;
    const int nbs = sb1 - sb0;
    const int wb0 = sb0 + (nbs * warp) / kGemvWeightWarps;
    const int nwb = sb0 + (nbs * (warp + 1)) / kGemvWeightWarps - wb0;   // <= BPW

    uint32_t xf[BPW][NH][8];
#pragma unroll
    for (int j = 0; j < BPW; ++j) gemv_load_x<NH>(p.x, p.K, p.T, g, q, (wb0 + j) * 64, j < nwb, xf[j]);

    // codes of rows g, g+8 for each block (reloaded for the next group right
    // after use); raw scale parts of the (row, block) pairs this lane owns:
    // rows {g, g+8} x blocks {q, q+4, ...}
    constexpr int kOwn = (BPW + 3) / 4;
    uint2 cg[BPW][2];
    int sq[2][kOwn];
    float sst[2][kOwn], smn[2][kOwn];
    auto load_codes = [&](int64_t n0, int j) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int64_t row = n0 + g + 8 * rr;
        cg[j][rr] = (j < nwb) ? __ldg(reinterpret_cast<const uint2*>(p.codes + row * row_bytes +
                                                                       (wb0 + j) * 32 + 8 * q))
                              : make_uint2(0, 0);
      }
    };
    auto load_scales = [&](int64_t n0) {
#pragma unroll
      for (int o = 0; o < kOwn; ++o) {
        const int j = q + 4 * o;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          sq[rr][o] = 0; sst[rr][o] = 0.f; smn[rr][o] = 0.f;
          if (j < nwb) {
            const int64_t si = (n0 + g + 8 * rr) * p.kb + wb0 + j;
            sq[rr][o] = __ldg(p.qscale + si);
            sst[rr][o] = __ldg(p.dq_step + (si >> 8));
            smn[rr][o] = __ldg(p.dq_mean + (si >> 8));
          }
        }
      }
    };

    int ng = pidx;
    if (ng < ngroups) {
      load_scales(static_cast<int64_t>(ng) * 16);
#pragma unroll
      for (int j = 0; j < BPW; ++j) load_codes(static_cast<int64_t>(ng) * 16, j);
    }
    for (; ng < ngroups; ng += p.pcta) {
      const int ngn = ng + p.pcta;
      const bool more = ngn < ngroups;
      const int64_t nn0 = static_cast<int64_t>(ngn) * 16;
      float sh[2][kOwn];
#pragma unroll
      for (int o = 0; o < kOwn; ++o)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
          sh[rr][o] = restore_scale(static_cast<int8_t>(sq[rr][o]), sst[rr][o], smn[rr][o]);
      if (more) load_scales(nn0);

      float acc[NH][4];
#pragma unroll
      for (int h = 0; h < NH; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
#pragma unroll
      for (int j = 0; j < BPW; ++j) {
        // block scales of rows g and g+8 from the lane of this quad owning block j
        const int src = (lane & ~3) | (j & 3);
        const float s0 = __shfl_sync(full, sh[0][j >> 2], src);
        const float s1 = __shfl_sync(full, sh[1][j >> 2], src);
        if (j < nwb) {
          const uint2 c0 = cg[j][0], c1 = cg[j][1];
          if (more) load_codes(nn0, j);
          float cb[NH][4];
#pragma unroll
          for (int h = 0; h < NH; ++h) cb[h][0] = cb[h][1] = cb[h][2] = cb[h][3] = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // bytes 2i and 2i+1 of the thread's 8 code bytes, rows g and g+8
            const uint32_t w0 = (i < 2) ? c0.x : c0.y;
            const uint32_t w1 = (i < 2) ? c1.x : c1.y;
            const uint32_t s = (i & 1) * 16;
            uint32_t a0, a1, a2, a3;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a0) : "r"(tbl_lane + (((w0 >> s) & 0xFFu) << 7)));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a2) : "r"(tbl_lane + (((w0 >> (s + 8)) & 0xFFu) << 7)));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a1) : "r"(tbl_lane + (((w1 >> s) & 0xFFu) << 7)));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a3) : "r"(tbl_lane + (((w1 >> (s + 8)) & 0xFFu) << 7)));
#pragma unroll
            for (int h = 0; h < NH; ++h)
              mma_bf16_16816(cb[h], a0, a1, a2, a3, xf[j][h][2 * i], xf[j][h][2 * i + 1]);
          }
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            acc[h][0] = fmaf(s0, cb[h][0], acc[h][0]);
            acc[h][1] = fmaf(s0, cb[h][1], acc[h][1]);
            acc[h][2] = fmaf(s1, cb[h][2], acc[h][2]);
            acc[h][3] = fmaf(s1, cb[h][3], acc[h][3]);
          }
        }
      }
      float* rb = red + (buf * kGemvWarps + warp) * 256;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const int t0 = 2 * q + 8 * h;
        rb[t0 * 16 + g] = acc[h][0];
        rb[(t0 + 1) * 16 + g] = acc[h][1];
        rb[t0 * 16 + g + 8] = acc[h][2];
        rb[(t0 + 1) * 16 + g + 8] = acc[h][3];
      }
      named_bar_sync(1, kGemvThreads);
      if (tid < 256) {
        const int tok = tid >> 4, row = tid & 15;
        if (tok < p.T) {
          const float* rs = red + buf * kGemvWarps * 256 + tok * 16 + row;
          float sum = 0.f;
#pragma unroll
          for (int w = 0; w < kGemvWarps; ++w) sum += rs[w * 256];
          const int64_t n = static_cast<int64_t>(ng) * 16 + row;
          if (p.ks == 1) p.y[static_cast<int64_t>(tok) * p.N + n] = __float2bfloat16_rn(sum);
          else p.partial[(static_cast<int64_t>(split) * p.T + tok) * p.N + n] = sum;
        }
      }
      buf ^= 1;
    }
  } else {
    // ---------------------------------------------------------- LoRA warp
    const bool active = (p.B != nullptr) && (split == p.ks - 1);
    const int nlb = active ? (p.rp >> 6) : 0;
    uint32_t uf[kGemvMaxLoraBlocks][NH][8];
#pragma unroll
    for (int j = 0; j < kGemvMaxLoraBlocks; ++j)
      gemv_load_x<NH>(p.us, p.rp, p.T, g, q, j * 64, j < nlb, uf[j]);
    uint4 bl[kGemvMaxLoraBlocks][2][2];
    auto load_rows = [&](int ng) {
      const int64_t n0 = static_cast<int64_t>(ng) * 16;
#pragma unroll
      for (int j = 0; j < kGemvMaxLoraBlocks; ++j)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int e0 = j * 64 + 16 * q;
          const __nv_bfloat16* src = p.B + (n0 + g + 8 * rr) * p.r + e0;
          bl[j][rr][0] = (j < nlb && e0 < p.r) ? __ldg(reinterpret_cast<const uint4*>(src)) : make_uint4(0, 0, 0, 0);
          bl[j][rr][1] = (j < nlb && e0 + 8 < p.r) ? __ldg(reinterpret_cast<const uint4*>(src + 8)) : make_uint4(0, 0, 0, 0);
        }
    };
    int ng = pidx;
    if (active && ng < ngroups) load_rows(ng);
    for (; ng < ngroups; ng += p.pcta) {
      uint4 b[kGemvMaxLoraBlocks][2][2];
#pragma unroll
      for (int j = 0; j < kGemvMaxLoraBlocks; ++j)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) { b[j][rr][0] = bl[j][rr][0]; b[j][rr][1] = bl[j][rr][1]; }
      if (active && ng + p.pcta < ngroups) load_rows(ng + p.pcta);
      float acc[NH][4];
#pragma unroll
      for (int h = 0; h < NH; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
      if (active) {
#pragma unroll
        for (int j = 0; j < kGemvMaxLoraBlocks; ++j) {
          if (j < nlb) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4& r0 = b[j][0][i >> 1];
              const uint4& r1 = b[j][1][i >> 1];
              const uint32_t a0 = (i & 1) ? r0.z : r0.x;
              const uint32_t a2 = (i & 1) ? r0.w : r0.y;
              const uint32_t a1 = (i & 1) ? r1.z : r1.x;
              const uint32_t a3 = (i & 1) ? r1.w : r1.y;
#pragma unroll
              for (int h = 0; h < NH; ++h)
                mma_bf16_16816(acc[h], a0, a1, a2, a3, uf[j][h][2 * i], uf[j][h][2 * i + 1]);
            }
          }
        }
      }
      float* rb = red + (buf * kGemvWarps + warp) * 256;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const int t0 = 2 * q + 8 * h;
        rb[t0 * 16 + g] = acc[h][0];
        rb[(t0 + 1) * 16 + g] = acc[h][1];
        rb[t0 * 16 + g + 8] = acc[h][2];
        rb[(t0 + 1) * 16 + g + 8] = acc[h][3];
      }
      named_bar_sync(1, kGemvThreads);
      buf ^= 1;
    }
  }
}

// y[t][n] = bf16(sum over k-splits of partial[s][t][n]), fixed order.
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float* __restrict__ partial, int ks,
                                                          int64_t tn, __nv_bfloat16* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait_primary();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= tn) return;
  float sum = 0.f;
  for (int s = 0; s < ks; ++s) sum += partial[static_cast<int64_t>(s) * tn + i];
  y[i] = __float2bfloat16_rn(sum);
}

}  // namespace qn
