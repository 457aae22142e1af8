// nf4_storage.cuh -- NF4 quantization with double quantization, and
// dequantization to bf16.  Memory-bound kernels; every rounding step is an
// explicit IEEE operation so the results are bit-identical to the CPU
// definition of the format.
//
// [QLoRA glossary, "Come funziona QLoRA": each weight a 4-bit code into 16
//  normal-quantile levels, one absmax scale per block of 64; block scales
//  quantized to 8 bits in blocks of 256.  NF4 snippet: normalize by the
//  block absmax, nearest level, restore as level x scale.]
#pragma once

#include "common.cuh"

namespace qn {

// Largest i with L[i] <= x, then the nearer of L[i], L[i+1] by the fp32
// distance |x - L|, the lower index on a tie.  Requires -1 <= x <= 1.
// The fp32 distance to the levels is strictly unimodal in the level index
// (adjacent levels are >= 0.07 apart, far above fp32 rounding at |x| <= 2),
// so the minimum over all 16 levels is at i or i + 1.
__device__ __forceinline__ uint32_t nearest_level(float x, const float* sL) {
  uint32_t i = (x >= sL[8]) ? 8u : 0u;
  i += (x >= sL[i + 4]) ? 4u : 0u;
  i += (x >= sL[i + 2]) ? 2u : 0u;
  i += (x >= sL[i + 1]) ? 1u : 0u;
  if (i < 15u) {
    const float d0 = fabsf(__fsub_rn(x, sL[i]));
    const float d1 = fabsf(__fsub_rn(x, sL[i + 1]));
    if (d1 < d0) i += 1u;
  }
  return i;
}

// First level.  Eight lanes per block of 64 weights: lane j of a group of 8
// holds elements 8j .. 8j+7 (one 16-byte load) and writes code bytes
// 4j .. 4j+3 (one 4-byte store; element 2i in the low nibble of byte i);
// a warp covers 4 blocks per pass and keeps kUnroll passes of loads in
// flight.  absmax_out receives the exact fp32 absmax of every block.
//
// The code of x = fl32(w / absmax) is found without the division where that
// is safe: x~ = fl32(w * fl32(1 / absmax)) is within 1.5e-7 of x, and away
// from the midpoints between adjacent levels (where the fp32 distance rule
// and the real-number one agree) the nearest level of x~ is that of x.  x~
// is binned by rint(64 x~) + 64; a bin holds at most one midpoint (they are
// >= 0.08 apart), so the code is the bin's code below its midpoint, plus one
// above it.  Within kEncodeMargin of a midpoint, or when 1 / absmax is not
// finite, the element takes the exact path: the IEEE division and
// nearest_level.
constexpr int kEncodeBins = 129;
constexpr int kEncodeBinTable = 256;     // bins 129..255 never match a finite |x| <= 1; they make any index safe
constexpr float kEncodeMargin = 1e-6f;

template <int kUnroll>
__global__ void __launch_bounds__(256) nf4_encode_kernel(const uint4* __restrict__ w8,
                                                         uint32_t* __restrict__ codes4,
                                                         float* __restrict__ absmax_out,
                                                         int64_t nblk, Levels lv) {
  __shared__ float sL[16];
  __shared__ float2 bins[kEncodeBinTable];     // {midpoint inside the bin or +inf, code below it}
  if (threadIdx.x < 16) sL[threadIdx.x] = lv.v[threadIdx.x];
  if (threadIdx.x < kEncodeBinTable) {
    const int t = threadIdx.x < kEncodeBins ? threadIdx.x : kEncodeBins - 1;
    const float lo = (static_cast<float>(t) - 64.5f) / 64.0f;
    const float hi = (static_cast<float>(t) - 63.5f) / 64.0f;
    int below = 0;
    float mid = __int_as_float(0x7f800000);
#pragma unroll
    for (int i = 0; i < 15; ++i) {
      const float m = 0.5f * (lv.v[i] + lv.v[i + 1]);
      if (m < lo) ++below;
      else if (m < hi) mid = m;
    }
    bins[threadIdx.x] = make_float2(mid, __int_as_float(below));
  }
  __syncthreads();
  const uint32_t lane = threadIdx.x & 31u;
  const int j = static_cast<int>(lane & 7u);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float magic = 12582912.0f;        // 1.5 * 2^23: adding it leaves rint(v) in the low mantissa bits
  for (int64_t b0 = warp * 4 * kUnroll; b0 < nblk; b0 += nwarps * 4 * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t b = b0 + 4 * u + (lane >> 3);
      v[u] = (b < nblk) ? __ldg(w8 + b * 8 + j) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t b = b0 + 4 * u + (lane >> 3);
      const uint32_t words[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      float w[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w[2 * e] = __uint_as_float(words[e] << 16);
        w[2 * e + 1] = __uint_as_float(words[e] & 0xFFFF0000u);
      }
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(w[e]));
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      const float r = __frcp_rn(a);
      // a zero or tiny absmax (1 / absmax not finite) is handled below; its
      // fast path runs on x = 0
      const float rf = (a > 0.0f && r < 3.0e38f) ? r : 0.0f;
      // fast path for all 8 elements, no branch; elements within the margin
      // of a midpoint are marked and redone exactly below
      uint32_t packed = 0, redo = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = __fmul_rn(w[e], rf);
        // |x| <= 1 + 2^-23 gives a bin in [0, 128]; the mask keeps any other
        // value (a non-finite weight) inside the table
        const int t = __float_as_int(__fmaf_rn(x, 64.0f, 64.0f + magic)) - __float_as_int(magic);
        const float2 bin = bins[t & (kEncodeBinTable - 1)];
        const uint32_t c = static_cast<uint32_t>(__float_as_int(bin.y)) + (x > bin.x ? 1u : 0u);
        packed |= c << (4 * e);
        redo |= (fabsf(x - bin.x) < kEncodeMargin ? 1u : 0u) << e;
      }
      if (!(a > 0.0f)) {
        packed = 0x77777777u;             // the zero level for an all-zero block
        redo = 0;
      } else if (!(r < 3.0e38f)) {
        redo = 0xFFu;                     // 1 / absmax not finite: every element exactly
      }
      if (redo) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if ((redo >> e) & 1u) {
            const uint32_t c = nearest_level(__fdiv_rn(w[e], a), sL);
            packed = (packed & ~(15u << (4 * e))) | (c << (4 * e));
          }
        }
      }
      if (b < nblk) {
        codes4[b * 8 + j] = packed;
        if (j == 0) absmax_out[b] = a;
      }
    }
  }
}

// Second level: one warp per group of 256 block scales.
// mean = fl32(S / c) with S the fp64 sum of the group (exact when the
// group's nonzero scales span less than 2^37, since every scale is a bf16
// value); d = fl32(s - mean); step = fl32(max|d| / 127);
// q = clamp(rint(fl32(d / step)), -127, 127), q = 0 when step = 0.
__global__ void __launch_bounds__(256) nf4_dq_kernel(const float* __restrict__ absmax,
                                                     int64_t nblk, int8_t* __restrict__ qscale,
                                                     float* __restrict__ dq_step,
                                                     float* __restrict__ dq_mean,
                                                     int64_t ngroups) {
  const uint32_t lane = threadIdx.x & 31u;
  const int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (g >= ngroups) return;
  const int64_t base = g * 256;
  const int64_t cnt64 = nblk - base < 256 ? nblk - base : 256;
  const int cnt = static_cast<int>(cnt64);
  float s[8];
  double sum = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = static_cast<int>(lane) + 32 * i;
    s[i] = (j < cnt) ? absmax[base + j] : 0.0f;
    sum += static_cast<double>(s[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  const float m = __double2float_rn(__ddiv_rn(sum, static_cast<double>(cnt)));
  float d[8];
  float cmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = static_cast<int>(lane) + 32 * i;
    d[i] = __fsub_rn(s[i], m);
    if (j < cnt) cmax = fmaxf(cmax, fabsf(d[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xFFFFFFFFu, cmax, o));
  const float step = __fdiv_rn(cmax, 127.0f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = static_cast<int>(lane) + 32 * i;
    if (j < cnt) {
      float q = 0.0f;
      if (step != 0.0f) {
        q = rintf(__fdiv_rn(d[i], step));
        q = fminf(fmaxf(q, -127.0f), 127.0f);
      }
      qscale[base + j] = static_cast<int8_t>(static_cast<int>(q));
    }
  }
  if (lane == 0) {
    dq_step[g] = step;
    dq_mean[g] = m;
  }
}

// Restored block scale: two separately rounded fp32 operations, no FMA.
__device__ __forceinline__ float restore_scale(int8_t q, float step, float mean) {
  return __fadd_rn(__fmul_rn(static_cast<float>(q), step), mean);
}

// Dequantization: each thread turns 4 code bytes (8 weights, inside one
// block of 64) into 8 bf16 values: bf16_rne(fl32(level[code] * s_hat)), one
// 16-byte store.  A warp takes 32 * kU consecutive 4-byte items per pass
// (lane l the items l, l + 32, ...), so each of its stores covers 512
// contiguous bytes (whole sectors); all loads of a pass are issued before
// any arithmetic.
template <int kU>
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint32_t* __restrict__ codes4,
                                                          const int8_t* __restrict__ qscale,
                                                          const float* __restrict__ dq_step,
                                                          const float* __restrict__ dq_mean,
                                                          uint4* __restrict__ out, int64_t n8,
                                                          Levels lv) {
  __shared__ float sL[16];
  if (threadIdx.x < 16) sL[threadIdx.x] = lv.v[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t i0 = warp * 32 * kU; i0 < n8; i0 += nwarps * 32 * kU) {
    uint32_t c[kU];
    int8_t q[kU];
    float st[kU], mn[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t i = i0 + 32 * u + lane;
      c[u] = 0;
      q[u] = 0;
      st[u] = 0.f;
      mn[u] = 0.f;
      if (i < n8) {
        const int64_t blk = i >> 3;
        c[u] = __ldg(codes4 + i);
        q[u] = __ldg(qscale + blk);
        st[u] = __ldg(dq_step + (blk >> 8));
        mn[u] = __ldg(dq_mean + (blk >> 8));
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t i = i0 + 32 * u + lane;
      if (i >= n8) break;
      const float sh = restore_scale(q[u], st[u], mn[u]);
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t byte = (c[u] >> (8 * j)) & 0xFFu;
        o[j] = pack_bf16x2(__fmul_rn(sL[byte & 15u], sh), __fmul_rn(sL[byte >> 4], sh));
      }
      out[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace qn
