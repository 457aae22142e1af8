// gemv.cuh -- decode-shape forward (1..16 tokens): the NF4 GEMV.
//
// [QLoRA glossary, "Come funziona QLoRA": the frozen layer dequantizes its
//  NF4 weights just before the matmul and adds the LoRA path's output.]
//
// y[t][n] = sum_b s_hat(n, b) * sum_{k in block b} x[t][k] * level[code(n, k)]
//         + sum_j us[t][j] * B[n][j]               (us = bf16(s * x A^T))
//
// HBM-bound: each packed code byte is read once.  Work layout:
//  * a CTA owns a contiguous range of 16-row units of W and all of K; its
//    work is cut into units of 16 rows x one k-range of 256 (four 64-weight
//    blocks), numbered k-range-major, and each warp takes a contiguous run of
//    units, so that its x fragments change only when its k-range does;
//  * every warp streams its units' codes through its own ring of shared-
//    memory stages: lane 0 requests each unit (16 rows x 128 bytes, one TMA
//    box) several units ahead, and the warp waits on that stage's barrier;
//    no barrier couples the warps in the main loop;
//  * mma.sync m16n8k16 with the 16 weight rows as the A operand and the
//    tokens as the B operand (x, in registers); inside a block the k order of
//    an MMA is permuted so that a thread's A values come from 8 consecutive
//    code bytes of its rows g and g + 8 and its x values from 16 consecutive
//    columns; both operands use the same permutation, so the sum is unchanged;
//  * a thread's accumulator rows are its own weight rows g and g + 8, so it
//    reads those rows' int8 block scales and double-quantization constants
//    itself when a unit starts and multiplies each block's fp32 partial by
//    its restored scale (constant over the block): the tensor core sees the
//    levels;
//  * a code byte becomes a bf16 pair (level[low nibble], level[high nibble])
//    through a 256-entry table stored once per lane: entry e of lane l sits at
//    byte e * 256 + l * 4 (no bank conflicts), so one byte permute that puts
//    the code byte in bits 8..15 and the lane's offset in bits 0..7 forms the
//    address;
//  * each unit's 16 x 8 partial tile is parked in shared memory; at the end
//    of a batch the tiles of a unit row are summed over k-ranges in k order,
//    the LoRA product is added (after the kernel that computes us, which this
//    one may overlap, has finished) and y is written.
// With LoRA, u = x A^T runs in the same launch: its first r / 8 CTAs take
// 8 rank rows each (the unit layout on bf16 weights) and count themselves
// done in a workspace counter that the other CTAs wait for (bounded) before
// their final step; the last CTA to exit resets the counters.
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
  // NF4 GEMV: CTA c owns 16-row units [c ru_q + min(c, ru_r), ...) (ru_q
  // units each, one more for the first ru_r CTAs), and the 256-entry table
  // byte -> (bf16(level[lo nibble]), bf16(level[hi nibble])) it stores per lane
  int ru_q, ru_r;
  uint32_t lut[256];
  // with LoRA: the first n_u CTAs compute u = x A^T (8 rank rows each) and
  // count themselves done in sync[0]; every CTA counts its exit in sync[1],
  // and the last one to exit sets both back to zero
  int n_u;
  unsigned int* sync;
  // sibling linears: u has ur columns (all groups' ranks); output rows from
  // lgstart[i] on use its columns i * lgcol .. + r (lgroups == 1: one group)
  int ur;
  int lgroups, lgcol;
  int64_t lgstart[4];
};

constexpr int kGemvTableBytes = 256 * 256;
constexpr int kGemvSmemBudget = 227 * 1024 - 1024;   // dynamic bytes


// NH = 1: up to 8 tokens; NH = 2: up to 16.
template <int NH>
struct GemvCfg {
  static constexpr int kWarps = NH == 1 ? 16 : 12;
  static constexpr int kThreads = kWarps * 32;
};


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

// x fragments of one k-range for token g (and g + 8): per block b, the 16
// consecutive columns 64 b + 16 q .. + 15 (8 words): the MMA's B operand
// (NF4 path) or A operand (bf16 path) under the in-block k permutation.
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

template <int NH>
struct GemvRing {
  static constexpr int kDepth = 3;                                // stages per warp
  static constexpr uint32_t kStageBytes = 16 * 128;               // one unit: 16 rows x 128 code bytes
  static constexpr uint32_t kWarpBytes = kDepth * kStageBytes;
};
// Double-quantization groups (256 consecutive block scales) that the block
// scales of `nru` 16-row units with kb blocks per row can touch.
__host__ __device__ constexpr int gemv_dq_groups(int nru, int kb) { return (nru * 16 * kb) / 256 + 2; }
// Row pitch of the restored fp32 block scales: kb floats plus 16 bytes, so
// that the rows g = 0..7 that a warp's 16-byte loads touch fall in distinct
// banks.
__host__ __device__ constexpr uint32_t gemv_scale_pitch(int kb) { return static_cast<uint32_t>(kb) * 4 + 16; }

// Dynamic shared memory of the NF4 GEMV, laid out from the shared-window
// address `base` of its first byte.  The lookup table starts at the next
// 64 KB boundary, so that one byte permute forms a lookup's whole address
// (table bits 16..31, code byte in bits 8..15, lane offset in bits 0..7);
// the warps' code rings fill the room below the table (1 KB-aligned, as the
// 128-byte swizzle wants) and continue above it; then come the barriers
// (W x D code stages, the scales' barrier, the abort flag), the batch's int8
// block scales, its groups' (step, mean) pairs, its restored fp32 block
// scales and its parked tiles.
struct GemvSmem {
  uint32_t tbl;      // offset of the table
  int nlow;          // warps whose ring lies below the table
  uint32_t ring_hi;  // offset of the first ring above the table
  uint32_t bars, qs, dq, sc, red, total;
};
template <int NH>
__host__ __device__ constexpr GemvSmem gemv_smem_layout(uint32_t base, int nkr, int ru_batch, int T) {
  constexpr int W = GemvCfg<NH>::kWarps;
  constexpr uint32_t RB = GemvRing<NH>::kWarpBytes;
  GemvSmem L{};
  const int kb = 4 * nkr;
  L.tbl = (0x10000u - (base & 0xFFFFu)) & 0xFFFFu;
  L.nlow = static_cast<int>(L.tbl / RB) < W ? static_cast<int>(L.tbl / RB) : W;
  L.ring_hi = L.tbl + kGemvTableBytes;
  L.bars = L.ring_hi + static_cast<uint32_t>(W - L.nlow) * RB;
  L.qs = L.bars + (static_cast<uint32_t>(W) * GemvRing<NH>::kDepth + 2) * 8;
  L.qs = (L.qs + 15u) & ~15u;
  L.dq = L.qs + static_cast<uint32_t>(ru_batch) * 16 * kb;
  L.sc = L.dq + static_cast<uint32_t>(gemv_dq_groups(ru_batch, kb)) * 8;
  L.sc = (L.sc + 15u) & ~15u;
  L.red = L.sc + static_cast<uint32_t>(ru_batch) * 16 * gemv_scale_pitch(kb);
  L.total = L.red + static_cast<uint32_t>(nkr) * ru_batch * 16 * T * 4;
  return L;
}
// The shared-window address of the dynamic shared memory that the host
// sizes the layout for (the 1 KB the hardware reserves at the bottom of a
// CTA's window); the kernel checks the layout it derives from its own
// address against the size it was given.
constexpr uint32_t kGemvHostBase = 1024;

// Sums a batch's parked tiles (16-row units) over the k-ranges in k order,
// adds the LoRA product, y = base + bf16(s u) B^T, and writes y.
__device__ __forceinline__ void gemv_finish16(const GemvParams& p, const float* red, int ru0, int nru, int nthreads) {
  const int T = p.T;
  const int outs = nru * 16 * T;
  for (int o = threadIdx.x; o < outs; o += nthreads) {
    const int t = o / (nru * 16);
    const int nl = o - t * (nru * 16);
    const int rul = nl >> 4, row = nl & 15;
    float sum = 0.f;
    for (int kr = 0; kr < p.nkr; ++kr) sum += red[(static_cast<int64_t>(kr * nru + rul) * 16 + row) * T + t];
    const int64_t n = static_cast<int64_t>(ru0) * 16 + nl;
    if (p.B) {
      int goff = 0;
      for (int gi = 1; gi < p.lgroups; ++gi)
        if (n >= p.lgstart[gi]) goff = gi * p.lgcol;
      const uint4* b8 = reinterpret_cast<const uint4*>(p.B + n * p.r);
      const uint4* u8 = reinterpret_cast<const uint4*>(p.us + static_cast<int64_t>(t) * p.rp + goff);
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

// The table word of code byte k (0..3) of `w` for this lane: `lk` holds the
// table's 64 KB-aligned address with lane * 4 in its low byte, and one byte
// permute puts byte k of w above the lane offset.
__device__ __forceinline__ uint32_t gemv_lookup(uint32_t w, uint32_t lk, int k) {
  return ld_shared_b32(__byte_perm(w, lk, 0x7604u | (static_cast<uint32_t>(k) << 4)));
}

// u = x A^T for rank rows 8 rg .. 8 rg + 7 (the LoRA path of a decode
// call): the unit layout of the NF4 GEMV on bf16 weights, each thread's 16
// weights of a block straight from global memory into registers; tokens are
// the MMA's A operand, the 8 rank rows its B operand.  Writes u (when asked)
// and bf16(s u).
template <int NH>
__device__ __forceinline__ void gemv_u_rows(const GemvParams& p, int rg, float* red) {
  constexpr int W = GemvCfg<NH>::kWarps;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int i0 = (warp * p.nkr) / W, i1 = ((warp + 1) * p.nkr) / W;
  uint32_t xf[NH][4][8];
  for (int kr = i0; kr < i1; ++kr) {
    gemv_load_x<NH>(p, kr, g, q, xf);
    GemvBf16Unit u;
    gemv_load_bf16_unit(p, static_cast<int64_t>(rg) * 8 + g, kr, q, u);
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
    gemv_park(red, kr, p.T, g, q, acc);
  }
  __syncthreads();
  // sum over the k-ranges in k order
  const int T = p.T;
  for (int o = tid; o < 8 * T; o += W * 32) {
    const int t = o >> 3, row = o & 7;
    float sum = 0.f;
    for (int kr = 0; kr < p.nkr; ++kr) sum += red[(kr * 8 + row) * T + t];
    const int n = rg * 8 + row;
    if (p.u_out) p.u_out[static_cast<int64_t>(t) * p.ur + n] = __float2bfloat16_rn(sum);
    p.us_out[static_cast<int64_t>(t) * p.us_ld + n] = __float2bfloat16_rn(__fmul_rn(p.s, sum));
  }
}

// Bounded wait until *ctr >= target (acquire, GPU scope).
__device__ __forceinline__ bool gemv_wait_count(const unsigned int* ctr, unsigned int target, volatile int* abort,
                                                unsigned int err_bit) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
  if (v >= target) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    __nanosleep(64);
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_error_word, err_bit);
      *abort = 1;
      return false;
    }
  }
}

// The NF4 GEMV.  A unit is 16 weight rows x one k-range of 256.  The 16
// rows are the MMA's A operand (m16n8k16) and the tokens its B operand:
// thread (g, q) looks up the A fragment from its own code bytes of rows g
// and g + 8, and scales the block partials of those rows by their restored
// block scales.  Each warp streams its units' codes through a ring of
// shared-memory stages: a unit (16 rows x 128 bytes, one TMA box) is
// requested kDepth units ahead and the warp waits on that stage's barrier
// (bounded).  A batch's int8 block scales arrive by one bulk copy, beside
// its first code requests, and are restored to fp32 once, before its units.
template <int NH>
__global__ void __launch_bounds__(GemvCfg<NH>::kThreads, 1)
    qlora_gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, GemvParams p) {
  constexpr int W = GemvCfg<NH>::kWarps;
  constexpr int D = GemvRing<NH>::kDepth;
  constexpr uint32_t SB = GemvRing<NH>::kStageBytes;
  constexpr uint32_t RB = GemvRing<NH>::kWarpBytes;
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  const uint32_t base = smem_u32(gemv_smem);
  const GemvSmem L = gemv_smem_layout<NH>(base, p.nkr, p.rg_batch, p.T);
  if (L.total > dynamic_smem_bytes() || (base & 1023u) != 0) {   // the same in every CTA
    if (threadIdx.x == 0) atomicOr(&g_error_word, ERR_GEMV_LAYOUT);
    return;
  }

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  if (static_cast<int>(blockIdx.x) < p.n_u) {
    // LoRA path: u for rank rows 8 blockIdx.x .. + 7, then count it done
    pdl_launch_dependents();
    if (tid < 8) {   // its A rows into L2 while the preceding kernel drains
      prefetch_l2_bulk(p.wb + (static_cast<int64_t>(blockIdx.x) * 8 + tid) * p.K, static_cast<uint32_t>(p.K * 2));
    }
    pdl_wait_primary();
    gemv_u_rows<NH>(p, blockIdx.x, reinterpret_cast<float*>(gemv_smem));
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      atomicAdd(p.sync, 1u);
      if (atomicAdd(p.sync + 1, 1u) == gridDim.x - 1) {
        atomicExch(p.sync, 0u);
        atomicExch(p.sync + 1, 0u);
      }
    }
    return;
  }
  const int cta = static_cast<int>(blockIdx.x) - p.n_u;
  const uint32_t ring_off = warp < L.nlow ? static_cast<uint32_t>(warp) * RB
                                          : L.ring_hi + static_cast<uint32_t>(warp - L.nlow) * RB;
  uint8_t* ring = gemv_smem + ring_off;
  const uint32_t ring_s = base + ring_off;
  uint64_t* full = reinterpret_cast<uint64_t*>(gemv_smem + L.bars) + warp * D;
  const uint32_t full_s = smem_u32(full);
  uint64_t* sbar = reinterpret_cast<uint64_t*>(gemv_smem + L.bars) + W * D;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gemv_smem + L.bars + (W * D + 1) * 8);
  float2* dq = reinterpret_cast<float2*>(gemv_smem + L.dq);
  const uint32_t qs_s = base + L.qs;
  const uint32_t sc_s = base + L.sc;
  const uint32_t red_s = base + L.red;

  if (lane == 0) {
    for (int j = 0; j < D; ++j) mbar_init(&full[j], 1);
    if (warp == 0) {
      mbar_init(sbar, 1);
      *abort_flag = 0;
      tma_prefetch_desc(&tm_codes);
    }
    fence_barrier_init();
  }
  pdl_launch_dependents();

  // this CTA's 16-row units of W
  const int ru_begin = cta * p.ru_q + min(cta, p.ru_r);
  const int ru_end = ru_begin + p.ru_q + (cta < p.ru_r ? 1 : 0);
  const int kb = p.kb;
  // As the first kernel of a call, while the preceding kernel drains, pull
  // this CTA's codes, int8 block scales and rows of B into L2 (contiguous
  // row ranges; codes 16 KB per request).
  if (p.wait_all) {
    const uint32_t row_bytes = static_cast<uint32_t>(p.K / 2);
    const uint32_t cn = static_cast<uint32_t>(ru_end - ru_begin) * 16 * row_bytes;
    const uint32_t nc = (cn + 16383u) >> 14;
    if (static_cast<uint32_t>(tid) < nc) {
      const uint32_t o = static_cast<uint32_t>(tid) << 14;
      prefetch_l2_bulk(p.codes + static_cast<int64_t>(ru_begin) * 16 * row_bytes + o, min(16384u, cn - o));
    } else if (static_cast<uint32_t>(tid) == nc) {
      prefetch_l2_bulk(p.qscale + static_cast<int64_t>(ru_begin) * 16 * kb,
                       static_cast<uint32_t>(ru_end - ru_begin) * 16 * kb);
    } else if (static_cast<uint32_t>(tid) == nc + 1 && p.B) {   // this CTA's rows of B
      prefetch_l2_bulk(p.B + static_cast<int64_t>(ru_begin) * 16 * p.r,
                       static_cast<uint32_t>(ru_end - ru_begin) * 16 * p.r * 2);
    }
  }

  // the table: entry e of lane l at byte e * 256 + l * 4 (one copy per lane:
  // no bank conflicts), four lanes' copies per 16-byte store
  {
    uint4* tw = reinterpret_cast<uint4*>(gemv_smem + L.tbl);
    for (int j = tid; j < 256 * 8; j += W * 32) {
      const uint32_t v = p.lut[j >> 3];
      tw[(j >> 3) * 16 + (j & 7)] = make_uint4(v, v, v, v);
    }
  }
  // as the first kernel of a call (launched to overlap the previous kernel's
  // tail), wait for the preceding work before reading any input
  if (p.wait_all) pdl_wait_primary();

  const uint32_t lk = (base + L.tbl) | (static_cast<uint32_t>(lane) << 2);
  // this thread's 8 code bytes of block b in a stage, row g: 128-byte rows,
  // 16-byte chunks XOR-swizzled by (row & 7); block b's offset is off0 ^ (b << 5)
  const uint32_t off0 = static_cast<uint32_t>(g) * 128 + ((static_cast<uint32_t>((q >> 1) ^ g) & 7u) << 4) +
                        8u * static_cast<uint32_t>(q & 1);
  const int T = p.T;
  const uint32_t spitch = gemv_scale_pitch(kb);
  // parked tile offsets: rows g and g + 8, tokens 8h + 2q and + 1
  uint32_t po[NH];
  bool pv0[NH], pv1[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const int t0 = 8 * h + 2 * q;
    po[h] = static_cast<uint32_t>(g * T + t0) * 4u;
    pv0[h] = t0 < T;
    pv1[h] = t0 + 1 < T;
  }
  const uint32_t po8 = static_cast<uint32_t>(8 * T) * 4u;

  int stage = 0;         // this warp's next ring stage and its phase parity
  uint32_t phase = 0;
  int pending = 0;       // copies still in flight when a wait gave up
  int batch = 0;
  bool ok = true;
  bool u_ready = false;
  for (int ru0 = ru_begin; ru0 < ru_end && ok; ru0 += p.rg_batch, ++batch) {
    const int nru = min(p.rg_batch, ru_end - ru0);
    const int units = p.nkr * nru;
    const int i0 = (warp * units) / W;
    int i1 = ((warp + 1) * units) / W;
    // the warp's first units, one request per lane (lanes 0 .. D-1)
    if (lane < D && i0 + lane < i1) {
      const int u = i0 + lane;
      const int kr = u / nru;
      int st = stage + lane;
      if (st >= D) st -= D;
      mbar_arrive_expect_tx(&full[st], SB);
      tma_load_2d(&tm_codes, &full[st], ring + st * SB, kr * 128, (ru0 + u - kr * nru) * 16);
    }
    // the unit requested next, and the unit processed next
    int kr_p = (i0 + D) / nru, ru_p = i0 + D - kr_p * nru;
    int kr_c = i0 / nru, ru_c = i0 - kr_c * nru;
    // the batch's block scales: rows ru0 * 16 .. + nru * 16, contiguous
    // (the previous batch's readers are past the barrier that ended it)
    const int64_t sbase = static_cast<int64_t>(ru0) * 16 * kb;
    if (tid == 0) {
      const uint32_t bytes = static_cast<uint32_t>(nru) * 16 * kb;
      mbar_arrive_expect_tx(sbar, bytes);
      bulk_copy_g2s(gemv_smem + L.qs, p.qscale + sbase, bytes, sbar);
    }
    const int64_t g_lo = sbase >> 8;
    const uint32_t sb_mod = static_cast<uint32_t>(sbase & 255);
    const int ng = static_cast<int>((sb_mod + static_cast<uint32_t>(nru) * 16 * kb - 1) >> 8) + 1;
    for (int j = tid; j < ng; j += W * 32) dq[j] = make_float2(__ldg(p.dq_step + g_lo + j), __ldg(p.dq_mean + g_lo + j));
    uint32_t xf[NH][4][8];
    int cur_kr = -1;
    if (i0 < i1) {
      gemv_load_x<NH>(p, kr_c, g, q, xf);
      cur_kr = kr_c;
    }
    // the groups' steps and means are written; the previous batch's tiles
    // are consumed
    __syncthreads();
    // restore the batch's block scales once: s = fl(fl(q * step) + mean);
    // warp w takes rows w, w + W, ..., lanes the blocks
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(sbar, batch & 1, abort_flag, ERR_GEMV_WAIT))) ok = false;
    if (ok) {
      for (int r = warp; r < nru * 16; r += W) {
        const uint32_t rq = static_cast<uint32_t>(r) * kb;
        for (int blk = lane; blk < kb; blk += 32) {
          const int8_t qv = static_cast<int8_t>(ld_shared_b32_v(qs_s + ((rq + blk) & ~3u)) >> (8 * ((rq + blk) & 3)));
          const float2 d = dq[(sb_mod + rq + blk) >> 8];
          st_shared_f32(sc_s + static_cast<uint32_t>(r) * spitch + static_cast<uint32_t>(blk) * 4u,
                        __fadd_rn(__fmul_rn(static_cast<float>(qv), d.x), d.y));
        }
      }
    }
    __syncthreads();
    if (!ok || *abort_flag) {
      ok = false;
      pending = max(0, min(D, i1 - i0));
      i1 = i0;   // skip the loop; the batch barrier below still runs
    }
    for (int i = i0; i < i1; ++i) {
      const int kr = kr_c, rul = ru_c;
      if (++ru_c == nru) { ru_c = 0; ++kr_c; }
      // restored scales of rows g and g + 8 for the unit's 4 blocks
      const uint32_t sa_s = sc_s + static_cast<uint32_t>(rul * 16 + g) * spitch + static_cast<uint32_t>(kr) * 16u;
      const float4 s0v = ld_shared_f4_v(sa_s);
      const float4 s8v = ld_shared_f4_v(sa_s + 8u * spitch);
      if (kr != cur_kr) {
        gemv_load_x<NH>(p, kr, g, q, xf);
        cur_kr = kr;
      }
      // warp-uniform: a lane whose wait gave up takes the whole warp out
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_at(full_s + stage * 8u, phase, abort_flag, ERR_GEMV_WAIT))) {
        ok = false;
        pending = min(D, i1 - i);
        break;
      }
      // rows g and g + 8, bytes 8q .. 8q + 7 of each block
      const uint32_t sa = ring_s + static_cast<uint32_t>(stage) * SB + off0;
      uint2 c0[4], c8[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        c0[b] = ld_shared_v2_v(sa ^ (static_cast<uint32_t>(b) << 5));
        c8[b] = ld_shared_v2_v((sa ^ (static_cast<uint32_t>(b) << 5)) + 1024u);
      }
      // the stage is refilled (async proxy) with the unit D ahead once every lane has read it
      fence_proxy_async_smem();
      __syncwarp();
      if (i + D < i1) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], SB);
          tma_load_2d(&tm_codes, &full[stage], ring + stage * SB, kr_p * 128, (ru0 + ru_p) * 16);
        }
        if (++ru_p == nru) { ru_p = 0; ++kr_p; }
      }
      if (++stage == D) {
        stage = 0;
        phase ^= 1u;
      }
      const float s0[4] = {s0v.x, s0v.y, s0v.z, s0v.w};
      const float s8[4] = {s8v.x, s8v.y, s8v.z, s8v.w};
      float acc[NH][4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float t[NH][4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t w0 = (m < 2) ? c0[b].x : c0[b].y;
          const uint32_t w8 = (m < 2) ? c8[b].x : c8[b].y;
          const int k0 = 2 * (m & 1);
          const uint32_t a0 = gemv_lookup(w0, lk, k0), a2 = gemv_lookup(w0, lk, k0 + 1);
          const uint32_t a1 = gemv_lookup(w8, lk, k0), a3 = gemv_lookup(w8, lk, k0 + 1);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            if (m == 0) mma_bf16_16816_z(t[h], a0, a1, a2, a3, xf[h][b][0], xf[h][b][1]);
            else mma_bf16_16816(t[h], a0, a1, a2, a3, xf[h][b][2 * m], xf[h][b][2 * m + 1]);
          }
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (b == 0) {
            acc[h][0] = s0[b] * t[h][0];
            acc[h][1] = s0[b] * t[h][1];
            acc[h][2] = s8[b] * t[h][2];
            acc[h][3] = s8[b] * t[h][3];
          } else {
            acc[h][0] = fmaf(s0[b], t[h][0], acc[h][0]);
            acc[h][1] = fmaf(s0[b], t[h][1], acc[h][1]);
            acc[h][2] = fmaf(s8[b], t[h][2], acc[h][2]);
            acc[h][3] = fmaf(s8[b], t[h][3], acc[h][3]);
          }
        }
      }
      // park the unit's 16 x (8 NH) tile
      const uint32_t rt = red_s + static_cast<uint32_t>(kr * nru + rul) * static_cast<uint32_t>(64 * T);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (pv0[h]) {
          st_shared_f32(rt + po[h], acc[h][0]);
          st_shared_f32(rt + po[h] + po8, acc[h][2]);
        }
        if (pv1[h]) {
          st_shared_f32(rt + po[h] + 4u, acc[h][1]);
          st_shared_f32(rt + po[h] + po8 + 4u, acc[h][3]);
        }
      }
    }
    // the batch's scales go back to the async proxy (next batch's copy)
    fence_proxy_async_smem();
    __syncthreads();
    if (!ok || *abort_flag) {
      ok = false;
      break;
    }
    if (p.n_u > 0 && !u_ready) {
      // the LoRA product needs all of u: wait (bounded) for the u CTAs
      if (tid == 0) gemv_wait_count(p.sync, static_cast<unsigned int>(p.n_u), abort_flag, ERR_GEMV_WAIT);
      __syncthreads();
      if (*abort_flag) {
        ok = false;
        break;
      }
      u_ready = true;
    }
    gemv_finish16(p, reinterpret_cast<const float*>(gemv_smem + L.red), ru0, nru, W * 32);
  }
  // after a wait gave up: let the requested copies land before exit
  if (!ok) {
    volatile int dummy = 0;
    if (lane == 0) {
      int st = stage;
      uint32_t ph = phase;
      for (int j = 0; j < pending; ++j) {
        mbar_wait_at(full_s + st * 8u, ph, &dummy, ERR_GEMV_WAIT);
        if (++st == D) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
    if (tid == 0) mbar_wait(sbar, batch & 1, &dummy, ERR_GEMV_WAIT);
  }
  // count this CTA's exit; the last one resets the counters for the next call
  if (p.n_u > 0) {
    __syncthreads();
    if (tid == 0 && atomicAdd(p.sync + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.sync, 0u);
      atomicExch(p.sync + 1, 0u);
    }
  }
}

}  // namespace qn
