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

// First level: one warp per block of 64 weights, several blocks in flight
// per warp.  Lane l holds elements 2l and 2l+1 (one bf16 pair) and writes
// byte l of the block's 32-byte code row (element 2l in the low nibble).
// absmax_out receives the exact fp32 absmax of every block.
template <int kUnroll>
__global__ void __launch_bounds__(256) nf4_encode_kernel(const uint32_t* __restrict__ w2,
                                                         uint8_t* __restrict__ codes,
                                                         float* __restrict__ absmax_out,
                                                         int64_t nblk, Levels lv) {
  __shared__ float sL[16];
  if (threadIdx.x < 16) sL[threadIdx.x] = lv.v[threadIdx.x];
  __syncthreads();
  const uint32_t lane = threadIdx.x & 31u;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t b0 = warp * kUnroll; b0 < nblk; b0 += nwarps * kUnroll) {
    uint32_t v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t b = b0 + u;
      v[u] = (b < nblk) ? __ldg(w2 + b * 32 + lane) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t b = b0 + u;
      if (b >= nblk) break;
      const float w0 = __uint_as_float(v[u] << 16);
      const float w1 = __uint_as_float(v[u] & 0xFFFF0000u);
      float a = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      uint32_t c0 = 7u, c1 = 7u;   // zero level for an all-zero block
      if (a > 0.0f) {
        c0 = nearest_level(__fdiv_rn(w0, a), sL);
        c1 = nearest_level(__fdiv_rn(w1, a), sL);
      }
      codes[b * 32 + lane] = static_cast<uint8_t>(c0 | (c1 << 4));
      if (lane == 0) absmax_out[b] = a;
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

// Dequantization: each thread turns 8 code bytes (16 weights, inside one
// block of 64) into 16 bf16 values: bf16_rne(fl32(level[code] * s_hat)).
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint2* __restrict__ codes8,
                                                          const int8_t* __restrict__ qscale,
                                                          const float* __restrict__ dq_step,
                                                          const float* __restrict__ dq_mean,
                                                          uint4* __restrict__ out, int64_t n16,
                                                          Levels lv) {
  __shared__ float sL[16];
  if (threadIdx.x < 16) sL[threadIdx.x] = lv.v[threadIdx.x];
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += stride) {
    const int64_t blk = i >> 2;
    const int64_t g = blk >> 8;
    const float sh = restore_scale(qscale[blk], __ldg(dq_step + g), __ldg(dq_mean + g));
    const uint2 c = __ldg(codes8 + i);
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t byte0 = (c.x >> (8 * j)) & 0xFFu;
      o[j] = pack_bf16x2(__fmul_rn(sL[byte0 & 15u], sh), __fmul_rn(sL[byte0 >> 4], sh));
      const uint32_t byte1 = (c.y >> (8 * j)) & 0xFFu;
      o[4 + j] = pack_bf16x2(__fmul_rn(sL[byte1 & 15u], sh), __fmul_rn(sL[byte1 >> 4], sh));
    }
    out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace qn
