// gemm_tc.cuh -- training-shape QLoRA linear on the 5th-generation tensor
// cores: a persistent tcgen05 GEMM whose B operand is the NF4 weight,
// decoded to bf16 in shared memory by dedicated warps just before the MMA.
//
// [QLoRA glossary, "Come funziona QLoRA": each frozen layer dequantizes its
//  NF4 weights to bfloat16 just before the matmul and adds the LoRA path;
//  backpropagation goes through the dequantized weights.  "Compromessi":
//  this dequantization on every forward and backward pass is the cost.]
//
// Two products share the kernel (GEMM notation D[m][n] = sum_k A[m][k] B[n][k]):
//   forward (kMode 0): y  = x  W_hat^T + (s u) B^T   A = x,  B op = W_hat (K-major)
//   dx      (kMode 1): dx = dy W_hat   + (s v) A     A = dy, B op = W_hat^T (MN-major)
// The LoRA product is one more k-block: A = the padded bf16(s u) or
// bf16(s v) from the rank-r kernel, B op = the LoRA matrix B (forward) or A
// (dx), both brought in by TMA with zero fill past rank r.
//
// CTA tile 256 (M) x BN (N), k-block 64, persistent over tiles.
//   warp 0      TMA producer: x / dy tiles (two 128-row boxes), LoRA slices
//   warp 1      MMA issuer (one thread) and TMEM owner
//   warps 4-7   epilogue: TMEM -> registers -> bf16 (or fp32) -> global
//   warps 8-15  decoders, two groups of 4 taking alternate k-blocks: each
//               thread turns one (weight row, 64-block) of codes into 128
//               bytes of the 128-byte-swizzled operand tile
// Pipeline: kStages smem stages (full / empty mbarriers; full counts the TMA
// arrival plus 128 decoder arrivals), two TMEM accumulators when BN = 128.
// Every wait is bounded (see mbar_wait).
#pragma once

#include "common.cuh"
#include "nf4_storage.cuh"

namespace qn {

struct GemmParams {
  const uint8_t* codes;     // [Nw, Kw/2]
  const int8_t* qscale;     // [Nw*Kw/64]
  const float* dq_step;
  const float* dq_mean;
  int64_t nw, kw;           // weight shape
  int64_t m, n, k;          // GEMM shape: forward (M, Nw, Kw), dx (M, Kw, Nw)
  int ksteps;               // k / 64
  int lora_steps;           // padded rank / 64 (0 without LoRA)
  int m_tiles, n_tiles;
  __nv_bfloat16* out;       // [m, n]
  float* outf;              // fp32 [m, n] output of the kF32Out instantiation
  Levels lv;
};

constexpr int kGemmThreads = 512;
constexpr int kBM = 256;

template <int BN>
struct GemmCfg {
  static constexpr int kStages = (BN == 128) ? 4 : 3;
  static constexpr int kAccStages = (BN == 128) ? 2 : 1;
  static constexpr int kAccCols = 2 * BN;                 // two 128-row halves
  static constexpr uint32_t kABytes = kBM * 128;          // 32 KB
  static constexpr uint32_t kBBytes = BN * 128;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kBarOffset = kStages * kStageBytes;
  static constexpr uint32_t kSmemBytes = kBarOffset + 256 + 1024;   // + barriers + alignment slack
};

// One decoder unit: 64 weights of one row and one 64-block, the raw inputs.
struct DecodeSrc {
  uint4 c0, c1;      // 32 code bytes
  int q;             // int8 block scale
  float step, mean;
  int valid;
};

__device__ __forceinline__ void decode_fetch(const GemmParams& p, int64_t row, int64_t kb,
                                             DecodeSrc& d) {
  d.valid = (row < p.nw) && (kb * 64 < p.kw);
  if (d.valid) {
    const uint4* src = reinterpret_cast<const uint4*>(p.codes + row * (p.kw >> 1) + kb * 32);
    d.c0 = __ldg(src);
    d.c1 = __ldg(src + 1);
    const int64_t si = row * (p.kw >> 6) + kb;
    d.q = __ldg(p.qscale + si);
    d.step = __ldg(p.dq_step + (si >> 8));
    d.mean = __ldg(p.dq_mean + (si >> 8));
  } else {
    d.c0 = d.c1 = make_uint4(0, 0, 0, 0);
    d.q = 0;
    d.step = 0.f;
    d.mean = 0.f;
  }
}

// Eight codes (one 32-bit word) -> eight bf16 (four 32-bit words) through
// byte tables: tl*/th* hold the low / high bytes of the 16 bf16 values
// bf16(level[c] * s_hat), four per register.
__device__ __forceinline__ uint4 decode_word(uint32_t w, uint32_t tl0, uint32_t tl1, uint32_t tl2,
                                             uint32_t tl3, uint32_t th0, uint32_t th1,
                                             uint32_t th2, uint32_t th3) {
  uint32_t out[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t sel = (h == 0) ? w : (w >> 16);        // four nibbles in the low 16 bits
    const uint32_t s3 = sel & 0x7777u;                    // index within a half table
    // byte mask: 0xFF where the nibble is >= 8 (sign-replicate of a 0x80 byte)
    const uint32_t msel = ((sel >> 3) & 0x1111u) | 0x8888u;
    const uint32_t msk = prmt_sign(0x00008000u, 0u, msel);
    const uint32_t la = __byte_perm(tl0, tl1, s3), lb = __byte_perm(tl2, tl3, s3);
    const uint32_t ha = __byte_perm(th0, th1, s3), hb = __byte_perm(th2, th3, s3);
    const uint32_t lo = (la & ~msk) | (lb & msk);
    const uint32_t hi = (ha & ~msk) | (hb & msk);
    out[2 * h] = __byte_perm(lo, hi, 0x5140u);
    out[2 * h + 1] = __byte_perm(lo, hi, 0x7362u);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// Decodes one unit into the 128-byte row `unit` of a swizzled operand tile.
__device__ __forceinline__ void decode_unit(const DecodeSrc& d, const float* sL, uint8_t* tile,
                                            int unit) {
  const float sh = restore_scale(static_cast<int8_t>(d.q), d.step, d.mean);
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__fmul_rn(sL[2 * i], sh), __fmul_rn(sL[2 * i + 1], sh));
  const uint32_t tl0 = __byte_perm(pk[0], pk[1], 0x6420u), th0 = __byte_perm(pk[0], pk[1], 0x7531u);
  const uint32_t tl1 = __byte_perm(pk[2], pk[3], 0x6420u), th1 = __byte_perm(pk[2], pk[3], 0x7531u);
  const uint32_t tl2 = __byte_perm(pk[4], pk[5], 0x6420u), th2 = __byte_perm(pk[4], pk[5], 0x7531u);
  const uint32_t tl3 = __byte_perm(pk[6], pk[7], 0x6420u), th3 = __byte_perm(pk[6], pk[7], 0x7531u);
  const uint32_t words[8] = {d.c0.x, d.c0.y, d.c0.z, d.c0.w, d.c1.x, d.c1.y, d.c1.z, d.c1.w};
  uint8_t* row = tile + unit * 128;
  const int sw = unit & 7;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint4 v = decode_word(words[m], tl0, tl1, tl2, tl3, th0, th1, th2, th3);
    *reinterpret_cast<uint4*>(row + ((m ^ sw) << 4)) = v;
  }
}

// kF32Out: the accumulators go to outf in fp32 (no LoRA k-block; the
// dropout backward adds its masked LoRA term and rounds once).  That
// instantiation runs beside the rank-r kernel launched before it and waits
// for it before exiting, so that its completion implies that kernel's.
template <int BN, int kMode, bool kF32Out = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,     // x or dy  [m, k]
                      const __grid_constant__ CUtensorMap tm_la,    // s*u or s*v [m, rp]
                      const __grid_constant__ CUtensorMap tm_lb,    // B [nw, r] or A [r, kw]
                      GemmParams p) {
  using Cfg = GemmCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOffset);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sL = reinterpret_cast<float*>(tmem_slot + 4);    // 16 floats

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1 + 128);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 16) sL[threadIdx.x] = p.lv.v[threadIdx.x];
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_la);
    tma_prefetch_desc(&tm_lb);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Only the LoRA slice (bf16(s u) or bf16(s v)) is produced by the kernel
  // that precedes this one; the TMA producer waits for it before loading
  // that slice, so the main loop overlaps the predecessor's tail.
  pdl_launch_dependents();

  const int nsteps = p.ksteps + p.lora_steps;
  const int ntiles = p.m_tiles * p.n_tiles;
  const int my_tiles = (ntiles > static_cast<int>(blockIdx.x))
                           ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;
  const int total_its = my_tiles * nsteps;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool waited = false;
      for (int t = 0; t < my_tiles && !*abort_flag; ++t) {
        const int tile = blockIdx.x + t * gridDim.x;
        const int m0 = (tile % p.m_tiles) * kBM;
        const int n0 = (tile / p.m_tiles) * BN;
        for (int ks = 0; ks < nsteps; ++ks, ++it) {
          const int stage = it % S;
          const uint32_t phase = (it / S) & 1;
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, ERR_GEMM_WAIT)) break;
          uint8_t* sa = smem + stage * Cfg::kStageBytes;
          uint8_t* sb = sa + Cfg::kABytes;
          if (ks < p.ksteps) {
            mbar_arrive_expect_tx(&full[stage], Cfg::kABytes);
            tma_load_2d(&tm_a, &full[stage], sa, ks * 64, m0);
            tma_load_2d(&tm_a, &full[stage], sa + 16384, ks * 64, m0 + 128);
          } else {
            const int lk = (ks - p.ksteps) * 64;
            if (!waited) {
              pdl_wait_primary();
              waited = true;
            }
            mbar_arrive_expect_tx(&full[stage], Cfg::kABytes + Cfg::kBBytes);
            tma_load_2d(&tm_la, &full[stage], sa, lk, m0);
            tma_load_2d(&tm_la, &full[stage], sa + 16384, lk, m0 + 128);
            if (kMode == 0) {
              tma_load_2d(&tm_lb, &full[stage], sb, lk, n0);
            } else {
#pragma unroll
              for (int a = 0; a < BN / 64; ++a) tma_load_2d(&tm_lb, &full[stage], sb + a * 8192, n0 + 64 * a, lk);
            }
          }
        }
      }
      // Drain: the last stages' copies must land before the CTA exits.
      const int issued = it;
      for (int j = (issued > S ? issued - S : 0); j < issued; ++j) {
        volatile int dummy = 0;
        mbar_wait(&full[j % S], (j / S) & 1, &dummy, ERR_GEMM_WAIT);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, kMode);
      const uint32_t lbo = (kMode == 0) ? 0u : 8192u;
      int it = 0;
      for (int t = 0; t < my_tiles && !*abort_flag; ++t) {
        const int acc = t % Cfg::kAccStages;
        const uint32_t acc_phase = (t / Cfg::kAccStages) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, ERR_GEMM_WAIT)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * Cfg::kAccCols;
        bool ok = true;
        for (int ks = 0; ks < nsteps; ++ks, ++it) {
          const int stage = it % S;
          const uint32_t phase = (it / S) & 1;
          if (!mbar_wait(&full[stage], phase, abort_flag, ERR_GEMM_WAIT)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * Cfg::kStageBytes);
          const uint32_t sb = sa + Cfg::kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = (kMode == 0) ? smem_desc_sw128(sb + kk * 32, lbo, 1024)
                                                : smem_desc_sw128(sb + kk * 2048, lbo, 1024);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t adesc = smem_desc_sw128(sa + h * 16384 + kk * 32, 0, 1024);
              umma_bf16_ss(d0 + h * BN, adesc, bdesc, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int wq = warp & 3;
    for (int t = 0; t < my_tiles; ++t) {
      const int tile = blockIdx.x + t * gridDim.x;
      const int m0 = (tile % p.m_tiles) * kBM;
      const int n0 = (tile / p.m_tiles) * BN;
      const int acc = t % Cfg::kAccStages;
      const uint32_t acc_phase = (t / Cfg::kAccStages) & 1;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, ERR_GEMM_WAIT)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int64_t row = m0 + h * 128 + wq * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + acc * Cfg::kAccCols + h * BN + c * 32, v);
          tmem_ld_wait();
          const int64_t col = n0 + c * 32;
          if constexpr (kF32Out) {
            if (row < p.m && col < p.n) {
              float4* dst = reinterpret_cast<float4*>(p.outf + row * p.n + col);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
            }
          } else if (row < p.m && col < p.n) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * p.n + col);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
              o.y = pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
              o.z = pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
              o.w = pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
              dst[j] = o;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ decoders
    const int grp = (warp - 8) >> 2;              // 0 or 1: takes iterations it % 2 == grp
    const int tid = threadIdx.x & 127;
    constexpr int kUnits = BN / 128;              // units per thread per k-block
    DecodeSrc cur[kUnits], nxt[kUnits];
    auto fetch = [&](int it, DecodeSrc (&d)[kUnits]) {
      const int tile = blockIdx.x + (it / nsteps) * gridDim.x;
      const int ks = it % nsteps;
      const int n0 = (tile / p.m_tiles) * BN;
#pragma unroll
      for (int i = 0; i < kUnits; ++i) {
        const int u = tid + 128 * i;
        if (ks >= p.ksteps) { d[i].valid = 0; continue; }
        int64_t row, kb;
        if (kMode == 0) { row = n0 + u; kb = ks; }
        else { row = static_cast<int64_t>(ks) * 64 + (u & 63); kb = n0 / 64 + (u >> 6); }
        decode_fetch(p, row, kb, d[i]);
      }
    };
    if (grp < total_its) fetch(grp, nxt);
    for (int it = grp; it < total_its; it += 2) {
#pragma unroll
      for (int i = 0; i < kUnits; ++i) cur[i] = nxt[i];
      if (it + 2 < total_its) fetch(it + 2, nxt);
      const int stage = it % S;
      const uint32_t phase = (it / S) & 1;
      if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, ERR_GEMM_WAIT)) break;
      const int ks = it % nsteps;
      if (ks < p.ksteps) {
        uint8_t* sb = smem + stage * Cfg::kStageBytes + Cfg::kABytes;
#pragma unroll
        for (int i = 0; i < kUnits; ++i) decode_unit(cur[i], sL, sb, tid + 128 * i);
        fence_proxy_async_smem();
      }
      mbar_arrive(&full[stage]);
    }
  }

  if constexpr (kF32Out) {
    if (threadIdx.x == 0) pdl_wait_primary();
  }
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace qn
