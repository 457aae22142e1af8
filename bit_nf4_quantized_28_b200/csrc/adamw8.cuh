// adamw8.cuh -- one AdamW step on the LoRA matrices with 8-bit states.
//
// [LoRA y QLoRA en Profundidad, "Optimizadores Paginados": QLoRA trains with
//  paged_adamw_8bit, Adam whose states are held in 8 bits ("Cálculo de
//  Memoria": a fraction of fp32 Adam's 8 bytes per parameter); Módulo 4:
//  QLoRA, 4.4: only the LoRA matrices train.  Paging is not built.]
//
// AdamW (decoupled weight decay), in fp32 one IEEE operation at a time:
//   m = b1 m0 + (1 - b1) g          v = b2 v0 + (1 - b2) g g
//   p1 = p (1 - lr wd)               p2 = p1 - ss (m / (sqrt(v) rb + eps))
// with the bias corrections in two host constants, ss = lr / (1 - b1^t) and
// rb = 1 / sqrt(1 - b2^t): one square root and one division per value.
// The states are stored per block of 256 values as one fp32 scale
// (absmax / 448) and one FP8 E4M3 code per value (value * (448 / absmax),
// or value / scale where that reciprocal overflows; round to nearest even,
// saturating; zero stored as +0).  The step reads m0, v0 from the codes,
// updates with the new m, v at full precision, then re-encodes them.  One warp owns one block: each lane 8 consecutive values (two
// 16-byte loads of p and g, 8 bytes of each code array), the block's absmax
// by shuffles.  HBM-bound: 4 + 4 + 1 + 1 bytes read and 4 + 1 + 1 (+ 2 for
// the bf16 copy) written per parameter, plus 8 bytes of scales per block.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace qn {

constexpr int kAdamBlock = 256;
constexpr int kAdamThreads = 128;     // 4 warps, one block of 256 values each per pass

struct AdamW8Params {
  float* p;                  // [n] fp32 master parameters, updated in place
  const float* g;            // [n] fp32 gradient
  uint8_t* mc;               // [n] E4M3 codes of m
  float* ms;                 // [ceil(n / 256)] scales of m
  uint8_t* vc;               // [n] E4M3 codes of v
  float* vs;                 // [ceil(n / 256)] scales of v
  __nv_bfloat16* pb;         // [n] bf16 copy of p, or null
  int64_t n;
  float b1, omb1, b2, omb2, step_size, rsqrt_bc2, decay, eps;
};

__device__ __forceinline__ float e4m3_value(uint8_t c) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3)));
}

__device__ __forceinline__ uint8_t e4m3_code(float x) {
  const uint8_t c = static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
  return (c & 0x7Fu) ? c : uint8_t{0};
}

__global__ void __launch_bounds__(kAdamThreads) adamw8_kernel(AdamW8Params p) {
  pdl_launch_dependents();
  pdl_wait_primary();
  const int lane = threadIdx.x & 31;
  const int64_t nblk = (p.n + kAdamBlock - 1) / kAdamBlock;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kAdamThreads) >> 5;
  for (int64_t b = (static_cast<int64_t>(blockIdx.x) * kAdamThreads + threadIdx.x) >> 5; b < nblk; b += nwarps) {
    const int64_t e0 = b * kAdamBlock + 8 * lane;
    const bool full = e0 + 8 <= p.n;
    float pv[8], gv[8];
    uint8_t mcv[8], vcv[8];
    if (full) {
      const float4* ps = reinterpret_cast<const float4*>(p.p + e0);
      const float4* gs = reinterpret_cast<const float4*>(p.g + e0);
      const float4 p0 = ps[0], p1 = ps[1], g0 = gs[0], g1 = gs[1];
      const uint2 mw = *reinterpret_cast<const uint2*>(p.mc + e0);
      const uint2 vw = *reinterpret_cast<const uint2*>(p.vc + e0);
      const float pa[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      const float ga[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        pv[j] = pa[j];
        gv[j] = ga[j];
        mcv[j] = static_cast<uint8_t>(((j < 4 ? mw.x : mw.y) >> (8 * (j & 3))) & 0xFFu);
        vcv[j] = static_cast<uint8_t>(((j < 4 ? vw.x : vw.y) >> (8 * (j & 3))) & 0xFFu);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool ok = e0 + j < p.n;
        pv[j] = ok ? p.p[e0 + j] : 0.f;
        gv[j] = ok ? p.g[e0 + j] : 0.f;
        mcv[j] = ok ? p.mc[e0 + j] : uint8_t{0};
        vcv[j] = ok ? p.vc[e0 + j] : uint8_t{0};
      }
    }
    const float msc = p.ms[b], vsc = p.vs[b];
    float mn[8], vn[8], pn[8];
    float am = 0.f, av = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float m0 = __fmul_rn(e4m3_value(mcv[j]), msc);
      const float v0 = __fmul_rn(e4m3_value(vcv[j]), vsc);
      const float g = gv[j];
      mn[j] = __fadd_rn(__fmul_rn(p.b1, m0), __fmul_rn(p.omb1, g));
      vn[j] = __fadd_rn(__fmul_rn(p.b2, v0), __fmul_rn(p.omb2, __fmul_rn(g, g)));
      const float p1 = __fmul_rn(pv[j], p.decay);
      const float den = __fadd_rn(__fmul_rn(__fsqrt_rn(vn[j]), p.rsqrt_bc2), p.eps);
      pn[j] = __fsub_rn(p1, __fmul_rn(p.step_size, __fdiv_rn(mn[j], den)));
      if (e0 + j < p.n) {
        am = fmaxf(am, fabsf(mn[j]));
        av = fmaxf(av, fabsf(vn[j]));
      }
    }
    // the parameters need no block-wide value: store them before the codes
    if (full) {
      float4* ps = reinterpret_cast<float4*>(p.p + e0);
      ps[0] = make_float4(pn[0], pn[1], pn[2], pn[3]);
      ps[1] = make_float4(pn[4], pn[5], pn[6], pn[7]);
      if (p.pb)
        *reinterpret_cast<uint4*>(p.pb + e0) = make_uint4(pack_bf16x2(pn[0], pn[1]), pack_bf16x2(pn[2], pn[3]),
                                                          pack_bf16x2(pn[4], pn[5]), pack_bf16x2(pn[6], pn[7]));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (e0 + j >= p.n) break;
        p.p[e0 + j] = pn[j];
        if (p.pb) p.pb[e0 + j] = __float2bfloat16_rn(pn[j]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
      av = fmaxf(av, __shfl_xor_sync(0xFFFFFFFFu, av, o));
    }
    const float sm = __fdiv_rn(am, 448.f), sv = __fdiv_rn(av, 448.f);
    // codes from x * (448 / absmax), or x / scale where that reciprocal overflows
    const float im = am > 0.f ? __fdiv_rn(448.f, am) : 1.f, iv = av > 0.f ? __fdiv_rn(448.f, av) : 1.f;
    const bool mfast = isfinite(im), vfast = isfinite(iv);
    uint32_t mw[2] = {0u, 0u}, vw[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t cm = sm > 0.f ? e4m3_code(mfast ? __fmul_rn(mn[j], im) : __fdiv_rn(mn[j], sm)) : 0u;
      const uint32_t cv = sv > 0.f ? e4m3_code(vfast ? __fmul_rn(vn[j], iv) : __fdiv_rn(vn[j], sv)) : 0u;
      mw[j >> 2] |= cm << (8 * (j & 3));
      vw[j >> 2] |= cv << (8 * (j & 3));
    }
    if (full) {
      *reinterpret_cast<uint2*>(p.mc + e0) = make_uint2(mw[0], mw[1]);
      *reinterpret_cast<uint2*>(p.vc + e0) = make_uint2(vw[0], vw[1]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (e0 + j >= p.n) break;
        p.mc[e0 + j] = static_cast<uint8_t>((mw[j >> 2] >> (8 * (j & 3))) & 0xFFu);
        p.vc[e0 + j] = static_cast<uint8_t>((vw[j >> 2] >> (8 * (j & 3))) & 0xFFu);
      }
    }
    if (lane == 0) {
      p.ms[b] = sm;
      p.vs[b] = sv;
    }
  }
}

}  // namespace qn
