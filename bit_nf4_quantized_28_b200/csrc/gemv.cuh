// gemv.cuh -- decode-shape forward (1..16 tokens): split-K NF4 GEMV.
//
// [QLoRA glossary, "Come funziona QLoRA": the frozen layer dequantizes its
//  NF4 weights just before the matmul and adds the LoRA path's output.]
//
// y[t][n] = sum_b s_hat(n, b) * sum_{k in block b} x[t][k] * level[code(n, k)]
//         + sum_j us[t][j] * B[n][j]               (us = bf16(s * x A^T))
//
// HBM-bound: each packed code byte is read once.  Layout of the work:
//  * the CTA walks groups of 16 weight rows; a producer warp streams each
//    group's code rows (this CTA's k-range) into a two-stage shared-memory
//    ring with bulk asynchronous copies (no multicast), so the loads of the
//    next group are in flight while the current one is decoded;
//  * mma.sync m16n8k16 with 16 weight rows as the A operand and the tokens
//    as the 8-column B operand (two column halves for 9..16 tokens);
//  * inside each 64-weight block the k order of an MMA is permuted so that a
//    thread's A values come from 8 consecutive code bytes of its row (one
//    64-bit shared load) and its x values from 16 consecutive columns; both
//    operands use the same permutation, so the sum is unchanged;
//  * a code byte becomes a bf16 pair (level[low nibble], level[high nibble])
//    through a 256-entry table stored once per lane (conflict-free loads);
//    entries are 256 bytes apart, so the byte-select permute that extracts a
//    code byte already yields its table offset;
//  * the block scale multiplies the block's fp32 partial product (the scale
//    is constant over the block), so the tensor core sees the levels;
//  * 14 weight warps each keep the x fragments of a fixed range of blocks in
//    registers; warp 14 computes the LoRA product for the same rows; each
//    warp parks its partial tile per group in shared memory, and the tiles
//    of up to 4 groups are summed in a fixed order after one barrier of the
//    15 compute warps (the producer never waits on it).
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
  int stage_stride;           // bytes between code rows in a stage
  __nv_bfloat16* y;           // [T, N] when ks == 1
  float* partial;             // [ks, T, N] when ks > 1
  Levels lv;
};

constexpr int kGemvWeightWarps = 14;
constexpr int kGemvLoraWarp = kGemvWeightWarps;          // warp 14
constexpr int kGemvProducerWarp = kGemvWeightWarps + 1;  // warp 15
constexpr int kGemvComputeWarps = kGemvWeightWarps + 1;
constexpr int kGemvThreads = 16 * 32;
constexpr int kGemvMaxLoraBlocks = 2;               // r <= 128
constexpr int kGemvTableStride = 256;               // bytes between table entries
constexpr int kGemvTableBytes = 256 * kGemvTableStride;
constexpr int kGemvGroupSlots = 4;                  // row groups summed per barrier
constexpr int kGemvRedBytes = kGemvGroupSlots * kGemvComputeWarps * 256 * 4;
constexpr int kGemvStages = 2;
constexpr int kGemvMaxSegBytes = 2304;              // <= 72 blocks of 32 code bytes per row
constexpr int kGemvMaxStageBytes = 16 * (kGemvMaxSegBytes + 128);
constexpr size_t kGemvSmemBytes = kGemvTableBytes + kGemvRedBytes + kGemvStages * kGemvMaxStageBytes + 64;

// Row stride of a code stage: at least `seg` bytes and congruent to 32 mod
// 128, which makes the 64-bit loads of 16 rows x 4 lanes conflict-free.
__host__ __device__ constexpr int gemv_stage_stride(int seg) { return seg + ((32 - seg) % 128 + 128) % 128; }

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

// Sums the partial tiles of `count` row groups (slots 0..count-1) over the
// compute warps in a fixed order and stores them; called by the 15 compute
// warps at the same points, between two barriers of those warps.
__device__ __forceinline__ void gemv_flush(const GemvParams& p, const float* red, int first_ng, int count,
                                           int split) {
  constexpr int kThreads = kGemvComputeWarps * 32;
  named_bar_sync(1, kThreads);
  for (int i = threadIdx.x; i < count * 256; i += kThreads) {
    const int slot = i >> 8, tok = (i >> 4) & 15, row = i & 15;
    if (tok >= p.T) continue;
    const float* rs = red + slot * kGemvComputeWarps * 256 + tok * 16 + row;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kGemvComputeWarps; ++w) sum += rs[w * 256];
    const int64_t n = static_cast<int64_t>(first_ng + slot * p.pcta) * 16 + row;
    if (p.ks == 1) p.y[static_cast<int64_t>(tok) * p.N + n] = __float2bfloat16_rn(sum);
    else p.partial[(static_cast<int64_t>(split) * p.T + tok) * p.N + n] = sum;
  }
  named_bar_sync(1, kThreads);
}

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int NH, int BPW>
__global__ void __launch_bounds__(kGemvThreads, 1) qlora_gemv_kernel(GemvParams p) {
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  uint32_t* tbl = reinterpret_cast<uint32_t*>(gemv_smem);                         // [256][64], lanes 0..31
  float* red = reinterpret_cast<float*>(gemv_smem + kGemvTableBytes);             // [4][15][16 tok][16 rows]
  uint8_t* stages = gemv_smem + kGemvTableBytes + kGemvRedBytes;                  // [2][16 rows][stride]
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + kGemvStages * kGemvMaxStageBytes);
  uint64_t* empty = full + kGemvStages;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;

  // byte -> (bf16(level[lo]), bf16(level[hi])), one copy per lane.
  for (int i = tid; i < 256 * 32; i += kGemvThreads) {
    const int b = i >> 5;
    tbl[b * (kGemvTableStride / 4) + (i & 31)] = pack_bf16x2(p.lv.v[b & 15], p.lv.v[b >> 4]);
  }
  if (tid == 0) {
    for (int s = 0; s < kGemvStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvWeightWarps);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  // Only the LoRA warp reads what the preceding kernel wrote (bf16(s u)); it
  // waits for it, the other warps start at once.
  pdl_launch_dependents();
  __syncthreads();

  const int split = blockIdx.x / p.pcta;
  const int pidx = blockIdx.x % p.pcta;
  const int ngroups = static_cast<int>(p.N >> 4);
  const int my_groups = pidx < ngroups ? (ngroups - 1 - pidx) / p.pcta + 1 : 0;
  const int64_t row_bytes = p.K >> 1;
  const int sb0 = split * p.split_blocks;
  const int sb1 = min(p.kb, sb0 + p.split_blocks);
  const int nbs = sb1 - sb0;
  const int seg = nbs * 32;
  const int stride = p.stage_stride;
  const unsigned fullmask = 0xFFFFFFFFu;

  if (warp == kGemvProducerWarp) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      for (int gi = 0; gi < my_groups; ++gi) {
        const int s = gi % kGemvStages;
        const uint32_t ph = (gi / kGemvStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, &abort_flag, ERR_GEMV_WAIT)) break;
        const int64_t n0 = static_cast<int64_t>(pidx + gi * p.pcta) * 16;
        uint8_t* dst = stages + s * kGemvMaxStageBytes;
        mbar_arrive_expect_tx(&full[s], 16u * seg);
        for (int rr = 0; rr < 16; ++rr)
          bulk_copy_g2s(dst + rr * stride, p.codes + (n0 + rr) * row_bytes + sb0 * 32, seg, &full[s]);
      }
      // the last copies must land before the CTA exits
      for (int gi = max(0, my_groups - kGemvStages); gi < my_groups; ++gi) {
        int none = 0;
        mbar_wait(&full[gi % kGemvStages], (gi / kGemvStages) & 1, &none, ERR_GEMV_WAIT);
      }
    }
    return;
  }

  int slot = 0, chunk_ng = pidx;
  if (warp < kGemvWeightWarps) {
    // ---------------------------------------------------------- weight warps
    const int wb = (nbs * warp) / kGemvWeightWarps;                 // first block, relative to sb0
    const int nwb = (nbs * (warp + 1)) / kGemvWeightWarps - wb;     // <= BPW

    uint32_t xf[BPW][NH][8];
#pragma unroll
    for (int j = 0; j < BPW; ++j) gemv_load_x<NH>(p.x, p.K, p.T, g, q, (sb0 + wb + j) * 64, j < nwb, xf[j]);

    // raw scale parts of the (row, block) pairs this lane owns:
    // rows {g, g+8} x blocks {q, q+4, ...}; loaded one group ahead
    constexpr int kOwn = (BPW + 3) / 4;
    int sq[2][kOwn];
    float sst[2][kOwn], smn[2][kOwn];
    auto load_scales = [&](int64_t n0) {
#pragma unroll
      for (int o = 0; o < kOwn; ++o) {
        const int j = q + 4 * o;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          sq[rr][o] = 0; sst[rr][o] = 0.f; smn[rr][o] = 0.f;
          if (j < nwb) {
            const int64_t si = (n0 + g + 8 * rr) * p.kb + sb0 + wb + j;
            sq[rr][o] = __ldg(p.qscale + si);
            sst[rr][o] = __ldg(p.dq_step + (si >> 8));
            smn[rr][o] = __ldg(p.dq_mean + (si >> 8));
          }
        }
      }
    };
    const uint32_t tbl_lane = smem_u32(tbl) + (lane << 2);
    const int code_off = g * stride + wb * 32 + 8 * q;

    if (my_groups > 0) load_scales(static_cast<int64_t>(pidx) * 16);
    for (int gi = 0; gi < my_groups; ++gi) {
      const int ng = pidx + gi * p.pcta;
      const bool more = gi + 1 < my_groups;
      float sh[2][kOwn];
#pragma unroll
      for (int o = 0; o < kOwn; ++o)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
          sh[rr][o] = restore_scale(static_cast<int8_t>(sq[rr][o]), sst[rr][o], smn[rr][o]);
      if (more) load_scales(static_cast<int64_t>(ng + p.pcta) * 16);

      const int s = gi % kGemvStages;
      mbar_wait(&full[s], (gi / kGemvStages) & 1, &abort_flag, ERR_GEMV_WAIT);
      const uint8_t* st = stages + s * kGemvMaxStageBytes + code_off;

      float acc[NH][4];
#pragma unroll
      for (int h = 0; h < NH; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
#pragma unroll
      for (int j = 0; j < BPW; ++j) {
        // block scales of rows g and g+8 from the lane of this quad owning block j
        const int src = (lane & ~3) | (j & 3);
        const float s0 = __shfl_sync(fullmask, sh[0][j >> 2], src);
        const float s1 = __shfl_sync(fullmask, sh[1][j >> 2], src);
        if (j < nwb) {
          const uint2 c0 = *reinterpret_cast<const uint2*>(st + j * 32);
          const uint2 c1 = *reinterpret_cast<const uint2*>(st + 8 * stride + j * 32);
          float cb[NH][4];
#pragma unroll
          for (int h = 0; h < NH; ++h) cb[h][0] = cb[h][1] = cb[h][2] = cb[h][3] = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // bytes 2i and 2i+1 of the thread's 8 code bytes, rows g and g+8;
            // byte b of a word moved to bits 8..15 (zeros elsewhere) = its table offset
            const uint32_t w0 = (i < 2) ? c0.x : c0.y;
            const uint32_t w1 = (i < 2) ? c1.x : c1.y;
            const uint32_t sel0 = 0x4404u | ((2 * (i & 1)) << 4), sel1 = 0x4404u | ((2 * (i & 1) + 1) << 4);
            uint32_t a0, a1, a2, a3;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a0) : "r"(tbl_lane + __byte_perm(w0, 0u, sel0)));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a2) : "r"(tbl_lane + __byte_perm(w0, 0u, sel1)));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a1) : "r"(tbl_lane + __byte_perm(w1, 0u, sel0)));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a3) : "r"(tbl_lane + __byte_perm(w1, 0u, sel1)));
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
      // this warp is done with the stage
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      float* rb = red + (slot * kGemvComputeWarps + warp) * 256;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const int t0 = 2 * q + 8 * h;
        rb[t0 * 16 + g] = acc[h][0];
        rb[(t0 + 1) * 16 + g] = acc[h][1];
        rb[t0 * 16 + g + 8] = acc[h][2];
        rb[(t0 + 1) * 16 + g + 8] = acc[h][3];
      }
      if (++slot == kGemvGroupSlots || !more) {
        gemv_flush(p, red, chunk_ng, slot, split);
        slot = 0;
        chunk_ng = ng + p.pcta;
      }
    }
  } else {
    // ---------------------------------------------------------- LoRA warp
    const bool active = (p.B != nullptr) && (split == p.ks - 1);
    const int nlb = active ? (p.rp >> 6) : 0;
    if (active) pdl_wait_primary();
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
    if (active && my_groups > 0) load_rows(pidx);
    for (int gi = 0; gi < my_groups; ++gi) {
      const int ng = pidx + gi * p.pcta;
      const bool more = gi + 1 < my_groups;
      uint4 b[kGemvMaxLoraBlocks][2][2];
#pragma unroll
      for (int j = 0; j < kGemvMaxLoraBlocks; ++j)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) { b[j][rr][0] = bl[j][rr][0]; b[j][rr][1] = bl[j][rr][1]; }
      if (active && more) load_rows(ng + p.pcta);
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
      float* rb = red + (slot * kGemvComputeWarps + warp) * 256;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const int t0 = 2 * q + 8 * h;
        rb[t0 * 16 + g] = acc[h][0];
        rb[(t0 + 1) * 16 + g] = acc[h][1];
        rb[t0 * 16 + g + 8] = acc[h][2];
        rb[(t0 + 1) * 16 + g + 8] = acc[h][3];
      }
      if (++slot == kGemvGroupSlots || !more) {
        gemv_flush(p, red, chunk_ng, slot, split);
        slot = 0;
        chunk_ng = ng + p.pcta;
      }
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
