// gemv.cuh -- decode-shape forward (1..16 tokens): split-K NF4 GEMV.
//
// [QLoRA glossary, "Come funziona QLoRA": the frozen layer dequantizes its
//  NF4 weights just before the matmul and adds the LoRA path's output.]
//
// y[t][n] = sum_b s_hat(n, b) * sum_{k in block b} x[t][k] * level[code(n, k)]
//         + sum_j us[t][j] * B[n][j]               (us = bf16(s * x A^T))
//
// HBM-bound: each packed code byte is read once.  Layout of the work:
//  * a CTA owns one k-range (split) of up to G consecutive groups of 16
//    weight rows, each with its own shared-memory stage and barrier.  One
//    thread fills a stage with three kinds of copies, none with multicast:
//    the group's code rows as tensor copies of 128 bytes x 16 rows each
//    (128-byte swizzle), the raw int8 scale codes of each row as a bulk
//    copy, and the step / mean entries as two more tensor copies;
//  * two groups are requested at the start and one more each time a group
//    lands, so the groups land in order while HBM stays busy; with more
//    groups than stages, a stage is refilled once every warp is done with it;
//  * the 16 warps each own a fixed range of 64-weight blocks of the k-range
//    and keep the matching x fragments in registers; each warp parks its
//    partial tile of every group in shared memory, and the tiles are summed
//    over the warps once, at the end, in warp order;
//  * mma.sync m16n8k16 with 16 weight rows as the A operand and the tokens
//    as the 8-column B operand (two column halves for 9..16 tokens);
//  * inside each block the k order of an MMA is permuted so that a thread's
//    A values come from 8 consecutive code bytes of its row (one 64-bit
//    shared load) and its x values from 16 consecutive columns; both operands
//    use the same permutation, so the sum is unchanged;
//  * a code byte becomes a bf16 pair (level[low nibble], level[high nibble])
//    through a 256-entry table stored once per lane: entry e of lane l sits at
//    byte e * 256 + l * 4 (no bank conflicts), so one byte permute that puts
//    the code byte in bits 8..15 and the lane's offset in bits 0..7 forms the
//    address;
//  * the block scale multiplies the block's fp32 partial product (the scale
//    is constant over the block), so the tensor core sees the levels.
// The LoRA product and the sum over k-splits happen in gemv_finalize_kernel
// when the layer has them.
#pragma once

#include "common.cuh"
#include "lora_small.cuh"
#include "nf4_storage.cuh"

namespace qn {

struct GemvParams {
  const int8_t* qscale;       // [N*K/64]
  const __nv_bfloat16* x;     // [T, K]
  int T;
  int64_t N, K;
  int kb;                     // K / 64
  int split_blocks;           // weight blocks per k-split (a multiple of 4)
  int ks;                     // k-splits
  int pcta;                   // CTAs per k-split
  int groups;                 // row groups per CTA (<= G of the kernel)
  int stages;                 // shared-memory stages (<= groups)
  int stage_bytes;            // bytes of one stage
  int code_bytes;             // bytes of a stage's code box (16 rows x chunks x 128)
  int qpitch;                 // bytes per row of a stage's scale codes
  int dq_box;                 // step / mean entries per stage
  int dq_pitch;               // bytes between a stage's step and mean boxes (a multiple of 128)
  int ring_bytes;             // bytes of all stages
  int wait_all;               // wait for the preceding kernel before any global access
  // LoRA product in the final step (one k-split only): y += us B^T for the
  // CTA's rows, B's rows staged in shared memory at lora_off
  const __nv_bfloat16* B;     // [N, r], or null
  const __nv_bfloat16* us;    // [T, rp] = bf16(s * x A^T)
  int r, rp;
  int lora_off;               // byte offset of the staged B rows in dynamic shared memory
  __nv_bfloat16* y;           // [T, N] (direct mode), or null
  float* partial;             // [ks, T, N] when y is null
  Levels lv;
};

// Tensor maps of the weight: codes [N, K/2] bytes in boxes of 128 bytes x
// 16 rows (128-byte swizzle), and the step / mean arrays as fp32 rows
// [1, ndq] (zero fill past the end).
struct GemvMaps {
  CUtensorMap codes;
  CUtensorMap step;
  CUtensorMap mean;
};

constexpr int kGemvWarps = 16;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvTableBytes = 256 * 256;
constexpr int kGemvSmemBudget = 227 * 1024 - 1024;   // dynamic bytes (1 KB goes to static shared memory)
constexpr int kGemvLead = 2;                        // groups requested ahead of the first one landing

// NH = 1: up to 8 tokens; NH = 2: up to 16.
template <int NH>
struct GemvCfg {
  static constexpr int kBPW = 64 / kGemvWarps;       // blocks per warp (x fragments in registers)
  static constexpr int kG = 6;                      // row groups per CTA
  static constexpr int kTokens = 8 * NH;
  static constexpr int kMaxSeg = kGemvWarps * kBPW * 32;   // code bytes per row and stage
  static constexpr int kTS = 17;                    // floats per token row of a reduction tile
};

// Bytes of one stage: the code boxes, then 16 rows of scale codes, then the
// step and mean boxes, each tensor-copy destination on a 128-byte boundary
// (at least one more chunk's worth after the code boxes: a warp's blocks
// past its range read up to one chunk beyond them, inside the stage).
__host__ __device__ constexpr int gemv_dq_pitch(int dq_box) { return (4 * dq_box + 127) / 128 * 128; }
__host__ __device__ constexpr int gemv_stage_bytes(int code_bytes, int qpitch, int dq_box) {
  return (code_bytes + (16 * qpitch + 2 * gemv_dq_pitch(dq_box) > 2048 ? 16 * qpitch + 2 * gemv_dq_pitch(dq_box)
                                                                         : 2048) +
          1023) /
         1024 * 1024;
}

// B fragments (tokens x 16 permuted k) of one 64-wide block for the mma: token
// g (+ 8 h), columns col0 + 16 q .. + 15.
template <int NH>
__device__ __forceinline__ void gemv_load_x(const __nv_bfloat16* base, int64_t ld, int T, int g,
                                            int q, int64_t col0, bool valid, uint32_t (&f)[NH][8]) {
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

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// First and one-past-last 16-byte-aligned offsets of row n's scale codes.
__host__ __device__ __forceinline__ int64_t gemv_q_lo(int64_t n, int kb, int sb0) {
  return (n * kb + sb0) & ~int64_t{15};
}
__host__ __device__ __forceinline__ int64_t gemv_q_hi(int64_t n, int kb, int sb1) {
  return (n * kb + sb1 + 15) & ~int64_t{15};
}
// First step / mean entry a stage holds for rows n0..n0+15 (a multiple of 4).
__host__ __device__ __forceinline__ int64_t gemv_dq_lo(int64_t n0, int kb, int sb0) {
  return ((n0 * kb + sb0) >> 8) & ~int64_t{3};
}

// Fills stage `stg` with row group `ng`; one whole warp issues the copies
// (lane c the code box of chunk c, lane 16 + r the scale codes of row r,
// lane 0 the step / mean boxes) and lane 0 posts the byte count, all on
// `full`.  A copy may complete before the count is posted: the phase cannot
// complete without lane 0's arrival.
__device__ __forceinline__ void gemv_fill_stage(const GemvParams& p, const GemvMaps& maps, uint8_t* stg,
                                                uint64_t* full, int64_t ng, int sb0, int sb1, int lane) {
  const int64_t n0 = ng * 16;
  const int chunks = p.code_bytes / 2048;
  uint8_t* qs = stg + p.code_bytes;
  if (lane == 0) fence_proxy_async_smem();
  __syncwarp();
  // one 128-byte x 16-row box per chunk: [chunk][row][128 bytes], swizzled
  for (int c = lane; c < chunks; c += 32)
    tma_load_2d(&maps.codes, full, stg + c * 2048, sb0 * 32 + c * 128, static_cast<int32_t>(n0));
  int64_t qbytes = 0;
  if (lane >= 16) {
    const int rr = lane - 16;
    const int64_t lo = gemv_q_lo(n0 + rr, p.kb, sb0), hi = gemv_q_hi(n0 + rr, p.kb, sb1);
    qbytes = hi - lo;
    bulk_copy_g2s(qs + rr * p.qpitch, p.qscale + lo, static_cast<uint32_t>(qbytes), full);
  }
  // total bytes of the stage, summed over the warp
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) qbytes += __shfl_xor_sync(0xFFFFFFFFu, qbytes, o);
  if (lane == 0) {
    mbar_arrive_expect_tx(full, static_cast<uint32_t>(p.code_bytes + 2 * 4 * p.dq_box + qbytes));
    uint8_t* dq = qs + 16 * p.qpitch;                       // 256-byte aligned: qpitch % 16 == 0
    const int32_t d0 = static_cast<int32_t>(gemv_dq_lo(n0, p.kb, sb0));
    tma_load_2d(&maps.step, full, dq, d0, 0);
    tma_load_2d(&maps.mean, full, dq + p.dq_pitch, d0, 0);
  }
}

// The table word of code byte k of `w` for this lane: lane4 holds lane * 4
// in its low byte, and one byte permute puts byte k of w above it.
__device__ __forceinline__ uint32_t gemv_lookup(const uint8_t* tbl, uint32_t w, uint32_t lane4, int k) {
  const uint32_t off = __byte_perm(w, lane4, 0x7604u | (static_cast<uint32_t>(k) << 4));
  return *reinterpret_cast<const uint32_t*>(tbl + off);
}

// Offset in a stage's code box of byte `o` (within the split) of row `r`:
// chunk-major [chunk][row][128 bytes], 16-byte units XOR-swizzled by row % 8.
__device__ __forceinline__ int gemv_code_off(int r, int o) {
  const int c = o >> 7, w = o & 127;
  return c * (16 * 128) + r * 128 + ((((w >> 4) ^ (r & 7))) << 4) + (w & 15);
}

// Sums the warps' partial tiles (red[warp][group][tok][TS], `tiles` floats
// per warp) in warp order, adds the LoRA product sum_j us[tok][j] Bs[row][j]
// when Bs is given (the CTA's B rows, [rows][r]), and writes the outputs: y
// (bf16) when given, else this split's slice of `partial`.
template <int NH>
__device__ __forceinline__ void gemv_finish(const float* red, int tiles, int outs, int T, int64_t N, int g0,
                                            int split, __nv_bfloat16* y, float* partial,
                                            const __nv_bfloat16* Bs, const __nv_bfloat16* us, int r, int rp) {
  using Cfg = GemvCfg<NH>;
  for (int i = threadIdx.x; i < outs; i += kGemvThreads) {
    const int row = i & 15, gt = i >> 4;                    // gt = group * T + tok
    const int gi = gt / T, tok = gt - gi * T;
    const float* src = red + gt * Cfg::kTS + row;
    float sum = 0.f;
#pragma unroll 8
    for (int w = 0; w < kGemvWarps; ++w) sum += src[w * tiles];
    if (Bs) {
      const uint4* b8 = reinterpret_cast<const uint4*>(Bs + (gi * 16 + row) * r);
      const uint4* u8 = reinterpret_cast<const uint4*>(us + static_cast<int64_t>(tok) * rp);
      float lora = 0.f;
      for (int c = 0; c < r / 8; ++c) {
        const uint4 bv = b8[c], uv = u8[c];
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          lora = fmaf(__uint_as_float(uw[e] << 16), __uint_as_float(bw[e] << 16), lora);
          lora = fmaf(__uint_as_float(uw[e] & 0xFFFF0000u), __uint_as_float(bw[e] & 0xFFFF0000u), lora);
        }
      }
      sum += lora;
    }
    const int64_t n = static_cast<int64_t>(g0 + gi) * 16 + row;
    if (y) y[static_cast<int64_t>(tok) * N + n] = __float2bfloat16_rn(sum);
    else partial[(static_cast<int64_t>(split) * T + tok) * N + n] = sum;
  }
}

template <int NH>
__global__ void __launch_bounds__(kGemvThreads, 1) qlora_gemv_kernel(const __grid_constant__ GemvMaps maps,
                                                                     GemvParams p) {
  using Cfg = GemvCfg<NH>;
  constexpr int BPW = Cfg::kBPW;
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  const uint8_t* tbl = gemv_smem;                                   // [256][64] words, 32 used
  uint8_t* ring = gemv_smem + kGemvTableBytes;                      // [stages][stage_bytes], 1024-aligned
  float* red = reinterpret_cast<float*>(ring + p.ring_bytes);       // [warp][group][tok][TS]
  const int red_floats = kGemvWarps * p.groups * p.T * Cfg::kTS;
  uint64_t* full = reinterpret_cast<uint64_t*>(red + ((red_floats + 1) & ~1));   // [stages]
  int* done = reinterpret_cast<int*>(full + p.stages);              // [stages] warps finished
  __nv_bfloat16* lora_b = reinterpret_cast<__nv_bfloat16*>(gemv_smem + p.lora_off);   // [rows][r]
  __shared__ __align__(8) uint64_t lora_bar;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  // MMA row g (and g + 8) holds weight row pg (and pg + 8) of the group:
  // rows 0, 2, 4, 6 for g = 0..3 and 1, 3, 5, 7 for g = 4..7, which makes the
  // swizzled code loads of each half warp hit 32 different banks
  const int pg = g < 4 ? 2 * g : 2 * g - 7;

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      done[s] = 0;
    }
    mbar_init(&lora_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&maps.codes);
    tma_prefetch_desc(&maps.step);
    tma_prefetch_desc(&maps.mean);
  }
  __syncthreads();
  pdl_launch_dependents();
  // As the first kernel of a call, wait for the preceding work before
  // touching its outputs; after our own rank-r kernel (which waits itself
  // before letting this kernel start) the inputs are already complete.
  if (p.wait_all) pdl_wait_primary();

  const int split = blockIdx.x / p.pcta;
  const int pidx = blockIdx.x % p.pcta;
  const int ngroups = static_cast<int>(p.N >> 4);
  const int g0 = pidx * p.groups;
  const int my_groups = max(0, min(p.groups, ngroups - g0));
  const int sb0 = split * p.split_blocks;
  const int sb1 = min(p.kb, sb0 + p.split_blocks);
  const int nbs = sb1 - sb0;
  const int nst = min(p.stages, my_groups);
  // what the final step needs, read now and held in registers
  int fin_T = p.T, fin_tiles = p.groups * p.T * Cfg::kTS;
  long long fin_N = p.N;
  __nv_bfloat16* fin_y = p.y;
  float* fin_partial = p.partial;
  asm volatile("" : "+r"(fin_T), "+r"(fin_tiles), "+l"(fin_N), "+l"(fin_y), "+l"(fin_partial));

  // The first kGemvLead groups are requested at once, before anything else
  // (the table below is built while they are in flight); group
  // gi + kGemvLead is requested as soon as group gi has landed, while stages
  // are still unused.  Requesting every stage at once makes them all land
  // together, late; this keeps the loads in order.
  if (warp < min(nst, kGemvLead))
    gemv_fill_stage(p, maps, ring + warp * p.stage_bytes, &full[warp], g0 + warp, sb0, sb1, lane);
  // the CTA's rows of B (contiguous in [N, r]) for the final step
  const bool lora = p.B != nullptr && my_groups > 0;
  if (lora && tid == kGemvThreads - 32) {
    const uint32_t bytes = static_cast<uint32_t>(my_groups * 16 * p.r * 2);
    mbar_arrive_expect_tx(&lora_bar, bytes);
    bulk_copy_g2s(lora_b, p.B + static_cast<int64_t>(g0) * 16 * p.r, bytes, &lora_bar);
  }

  // byte -> (bf16(level[lo]), bf16(level[hi])), one copy per lane; each
  // thread writes four lanes' copies of one entry at once
  {
    uint4* t128 = reinterpret_cast<uint4*>(gemv_smem);
    for (int i = tid; i < 256 * 8; i += kGemvThreads) {
      const int b = i >> 3;
      const uint32_t v = pack_bf16x2(p.lv.v[b & 15], p.lv.v[b >> 4]);
      t128[b * 16 + (i & 7)] = make_uint4(v, v, v, v);
    }
  }

  const int wb = (nbs * warp) / kGemvWarps;                 // first block, relative to sb0
  const int nwb = (nbs * (warp + 1)) / kGemvWarps - wb;     // <= BPW

  // x fragments of the warp's blocks (zero past nwb: those blocks add 0)
  uint32_t xf[BPW][NH][8];
#pragma unroll
  for (int j = 0; j < BPW; ++j)
    gemv_load_x<NH>(p.x, p.K, p.T, g, q, static_cast<int64_t>(sb0 + wb + j) * 64, j < nwb, xf[j]);

  // this lane's code offsets in a stage: rows pg and pg + 8 (the same
  // swizzle), 8 bytes at 32 (wb + j) + 8 q; blocks past nbs read other bytes
  int coff[BPW];
#pragma unroll
  for (int j = 0; j < BPW; ++j) coff[j] = gemv_code_off(pg, (wb + j) * 32 + 8 * q);

  __syncthreads();      // the table is complete
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
  const unsigned fullmask = 0xFFFFFFFFu;
  float* rw = red + warp * p.groups * p.T * Cfg::kTS;       // this warp's tiles

  int s = 0;
  uint32_t ph = 0;
  bool ok = true;
#pragma unroll 1
  for (int gi = 0; gi < my_groups; ++gi) {
    uint8_t* stg = ring + s * p.stage_bytes;
    if (!mbar_wait(&full[s], ph, &abort_flag, ERR_GEMV_WAIT)) { ok = false; break; }
    {
      const int nx = gi + kGemvLead;
      if (nx < nst && (nx % kGemvWarps) == warp)
        gemv_fill_stage(p, maps, ring + nx * p.stage_bytes, &full[nx], g0 + nx, sb0, sb1, lane);
    }
    // block scales of rows pg and pg + 8 for block q of the warp's range
    float sh0 = 0.f, sh1 = 0.f;
    if (q < nwb) {
      const uint8_t* qs = stg + p.code_bytes;
      const float* dq = reinterpret_cast<const float*>(qs + 16 * p.qpitch);
      const float* dm = reinterpret_cast<const float*>(qs + 16 * p.qpitch + p.dq_pitch);
      const int64_t n0 = static_cast<int64_t>(g0 + gi) * 16;
      const int64_t n = n0 + pg;
      const int64_t dlo = gemv_dq_lo(n0, p.kb, sb0);
      const int b = sb0 + wb + q;                             // absolute block in the row
      const int64_t i0 = n * p.kb + b, i8 = (n + 8) * p.kb + b;
      const int d0 = static_cast<int>((i0 >> 8) - dlo), d8 = static_cast<int>((i8 >> 8) - dlo);
      sh0 = restore_scale(static_cast<int8_t>(qs[pg * p.qpitch + static_cast<int>(i0 - gemv_q_lo(n, p.kb, sb0))]),
                          dq[d0], dm[d0]);
      sh1 = restore_scale(
          static_cast<int8_t>(qs[(pg + 8) * p.qpitch + static_cast<int>(i8 - gemv_q_lo(n + 8, p.kb, sb0))]),
          dq[d8], dm[d8]);
    }
    float acc[NH][4];
#pragma unroll
    for (int h = 0; h < NH; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      // blocks past nwb read other bytes of the stage; their x fragments and
      // scales are zero, so they add nothing
      const int src = (lane & ~3) | j;
      const float s0 = __shfl_sync(fullmask, sh0, src);
      const float s1 = __shfl_sync(fullmask, sh1, src);
      const uint2 c0 = *reinterpret_cast<const uint2*>(stg + coff[j]);
      const uint2 c1 = *reinterpret_cast<const uint2*>(stg + coff[j] + 8 * 128);
      float cb[NH][4];
#pragma unroll
      for (int h = 0; h < NH; ++h) cb[h][0] = cb[h][1] = cb[h][2] = cb[h][3] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // bytes 2i and 2i+1 of the thread's 8 code bytes, rows g and g+8
        const uint32_t w0 = (i < 2) ? c0.x : c0.y;
        const uint32_t w1 = (i < 2) ? c1.x : c1.y;
        const int k0 = 2 * (i & 1), k1 = k0 + 1;
        const uint32_t a0 = gemv_lookup(tbl, w0, lane4, k0);
        const uint32_t a2 = gemv_lookup(tbl, w0, lane4, k1);
        const uint32_t a1 = gemv_lookup(tbl, w1, lane4, k0);
        const uint32_t a3 = gemv_lookup(tbl, w1, lane4, k1);
#pragma unroll
        for (int h = 0; h < NH; ++h) mma_bf16_16816(cb[h], a0, a1, a2, a3, xf[j][h][2 * i], xf[j][h][2 * i + 1]);
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        acc[h][0] = fmaf(s0, cb[h][0], acc[h][0]);
        acc[h][1] = fmaf(s0, cb[h][1], acc[h][1]);
        acc[h][2] = fmaf(s1, cb[h][2], acc[h][2]);
        acc[h][3] = fmaf(s1, cb[h][3], acc[h][3]);
      }
    }
    // this warp's partial tile of the group: rw[group][tok][row]
    float* rb = rw + gi * p.T * Cfg::kTS;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const int t0 = 2 * q + 8 * h;
      if (t0 < p.T) {
        rb[t0 * Cfg::kTS + pg] = acc[h][0];
        rb[t0 * Cfg::kTS + pg + 8] = acc[h][2];
      }
      if (t0 + 1 < p.T) {
        rb[(t0 + 1) * Cfg::kTS + pg] = acc[h][1];
        rb[(t0 + 1) * Cfg::kTS + pg + 8] = acc[h][3];
      }
    }
    // more groups than stages: the last warp done with this stage refills it
    // with the group `stages` later
    if (gi + p.stages < my_groups) {
      __syncwarp();
      int prev = 0;
      if (lane == 0) {
        __threadfence_block();
        prev = atomicAdd(&done[s], 1);
        if (prev == kGemvWarps - 1) done[s] = 0;
      }
      prev = __shfl_sync(fullmask, prev, 0);
      if (prev == kGemvWarps - 1) gemv_fill_stage(p, maps, stg, &full[s], g0 + gi + p.stages, sb0, sb1, lane);
    }
    if (++s == p.stages) { s = 0; ph ^= 1; }
  }

  // With a LoRA path this kernel did not wait for the rank-r kernel before
  // it (only the inputs of the call are read here).  Wait now, before
  // finishing, so that this kernel's completion implies that kernel's, which
  // the finalize kernel after it relies on for us.
  if (!p.wait_all) pdl_wait_primary();
  // sum the warps' tiles in warp order (and add the LoRA product)
  __syncthreads();
  if (lora && !mbar_wait(&lora_bar, 0, &abort_flag, ERR_GEMV_WAIT)) ok = false;
  if (!ok) return;
  gemv_finish<NH>(red, fin_tiles, my_groups * 16 * fin_T, fin_T, fin_N, g0, split, fin_y, fin_partial,
                  lora ? lora_b : nullptr, p.us, p.r, p.rp);
}

// y[t][n] = bf16(sum over k-splits of partial[s][t][n] + sum_j us[t][j] B[n][j]),
// in a fixed order; us = bf16(s * x A^T) [T, rp], B [N, r] (r == 0: no LoRA).
// One thread per output (t, n); every load it makes is independent.
constexpr int kFinalizeThreads = 256;

__global__ void __launch_bounds__(kFinalizeThreads) gemv_finalize_kernel(
    const float* __restrict__ partial, int ks, int T, int64_t N, const __nv_bfloat16* __restrict__ us,
    int rp, const __nv_bfloat16* __restrict__ B, int r, __nv_bfloat16* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait_primary();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kFinalizeThreads + threadIdx.x;
  if (i >= static_cast<int64_t>(T) * N) return;
  const int t = static_cast<int>(i / N);
  const int64_t n = i - static_cast<int64_t>(t) * N;
  // the k-split partials, eight independent loads at a time, summed in order
  float sum = 0.f;
  for (int s0 = 0; s0 < ks; s0 += 8) {
    float part[8];
#pragma unroll
    for (int s = 0; s < 8; ++s)
      part[s] = s0 + s < ks ? partial[(static_cast<int64_t>(s0 + s) * T + t) * N + n] : 0.f;
#pragma unroll
    for (int s = 0; s < 8; ++s) sum += part[s];
  }
  float lora = 0.f;
  if (r > 0) {
    const uint4* brow = reinterpret_cast<const uint4*>(B + n * r);
    const uint4* urow = reinterpret_cast<const uint4*>(us + static_cast<int64_t>(t) * rp);
    uint4 bv[kMaxRank / 8], uv[kMaxRank / 8];
#pragma unroll
    for (int c = 0; c < kMaxRank / 8; ++c) {
      bv[c] = make_uint4(0, 0, 0, 0);
      uv[c] = bv[c];
      if (c < r / 8) {
        bv[c] = __ldg(brow + c);
        uv[c] = __ldg(urow + c);
      }
    }
#pragma unroll
    for (int c = 0; c < kMaxRank / 8; ++c) {
      const uint32_t bw[4] = {bv[c].x, bv[c].y, bv[c].z, bv[c].w};
      const uint32_t uw[4] = {uv[c].x, uv[c].y, uv[c].z, uv[c].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lora = fmaf(__uint_as_float(uw[e] << 16), __uint_as_float(bw[e] << 16), lora);
        lora = fmaf(__uint_as_float(uw[e] & 0xFFFF0000u), __uint_as_float(bw[e] & 0xFFFF0000u), lora);
      }
    }
  }
  y[i] = __float2bfloat16_rn(sum + lora);
}

}  // namespace qn
