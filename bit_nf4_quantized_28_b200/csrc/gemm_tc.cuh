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
// CTA tile 256 (M) x 256 (N), k-block 64, persistent over tiles.  The CTAs
// of a thread-block cluster (kC = 1, 2 or 4 of them) take kC consecutive
// M-tiles of the same N-tile, so they need the same decoded B tile at every
// k-block: each CTA decodes 1/kC of it and sends its rows to the others with
// bulk shared-to-shared copies (no multicast), so a weight tile is decoded
// once per cluster instead of once per CTA.
//   warp 0      TMA producer: x / dy tiles (two 128-row boxes), LoRA slices
//   warp 1      MMA issuer (one thread) and TMEM owner
//   warp 2      TMA producer of this CTA's share of the packed codes, into a
//               ring of its own that runs ahead of the decoders
//   warps 4-7   epilogue: TMEM -> registers -> bf16 (or fp32) -> global
//   warps 8-15  decoders (all 8, or 6 with clusters of 4), in groups taking
//               k-blocks in turn: a thread turns one (weight row, 64-block)
//               unit of codes, read from the code ring, into 128 bytes of the
//               128-byte-swizzled operand tile
// Barriers per operand stage: afull (TMA of A), bfull (every local decoder
// thread of the k-block, after its own proxy fence, the MMA thread's post of
// the bytes the other CTAs send, and those bytes), empty (one multicast
// commit from each CTA's MMA: the stage is free in every CTA of the cluster;
// the last stages' commits are waited for before the CTA exits, so that none
// reaches a CTA that has left).  Every wait is bounded (see mbar_wait).
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
  // forward of sibling linears: output rows from lgstart[i] on take their
  // LoRA block from columns i * lgcol of s*u (lgroups == 1: one group)
  int lgroups, lgcol;
  int64_t lgstart[4];
  int m_tiles, n_tiles;
  int mc_tiles;             // cluster M-tiles: ceil(m_tiles / kC)
  __nv_bfloat16* out;       // [m, n]
  float* outf;              // fp32 [m, n] output of the kF32Out instantiation
  Levels lv;
};

constexpr int kGemmThreads = 512;
constexpr int kBM = 256;
constexpr int kBN = 256;

template <int kC>
struct GemmCfg {
  static constexpr int kStages = 3;
  static constexpr uint32_t kABytes = kBM * 128;          // 32 KB
  static constexpr uint32_t kBBytes = kBN * 128;          // 32 KB
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kNU = 256 / kC;                    // units a CTA decodes per k-block
  static constexpr int kU = kC == 1 ? 2 : 1;              // units per decoder thread per k-block
  static constexpr int kNT = kNU / kU;                    // decoder threads per k-block
  // Decoder groups take k-blocks in turn.  No more groups than operand
  // stages: a group then never reaches a stage's empty barrier two phases
  // ahead of it (which its parity test could not tell from one phase behind).
  static constexpr int kG = (256 / kNT) < kStages ? (256 / kNT) : kStages;
  static constexpr int kDecWarps = kNT / 32;              // decoder warps per k-block
  static constexpr int kDecoders = kG * kDecWarps;        // decoder warps in use (of warps 8-15)
  // code stages: a multiple of the groups, so that each is read by one group
  static constexpr int kCStages = kC == 1 ? 4 : 6;
  static constexpr uint32_t kCBytes = 8192 / kC;          // this CTA's codes of one k-block
  static constexpr uint32_t kCPitch = 128 / kC;           // dx: bytes per weight row in a code stage
  static constexpr uint32_t kCodeOff = kStages * kStageBytes;
  static constexpr uint32_t kBarOff = kCodeOff + kCStages * kCBytes;
  static constexpr uint32_t kSmemBytes = kBarOff + 512 + 1024;   // + barriers + alignment slack
  static constexpr uint32_t kIncoming = (kC - 1) * kNU * 128;    // bytes the other CTAs send per k-block
  static_assert(kG <= kStages, "a decoder group must not run a whole ring ahead");
  static_assert(kCStages % kG == 0, "each code stage is read by one decoder group");
  static_assert(kDecoders <= 8, "decoders are warps 8-15");
};

// Inputs of one unit's block scale (zero for a unit past the weight).
struct ScaleSrc {
  int q;
  float step, mean;
};

// Weight row and 64-block of unit u (0..255) of the B tile at k-step ks of
// the N-tile starting at n0.  Forward: unit u is weight row n0 + u at block
// ks.  dx: weight row 64 ks + (u mod 64), block n0 / 64 + u / 64 (the tile's
// k runs along weight rows).
template <int kMode>
__device__ __forceinline__ void unit_coords(int u, int ks, int64_t n0, int64_t& row, int64_t& kb) {
  if (kMode == 0) {
    row = n0 + u;
    kb = ks;
  } else {
    row = static_cast<int64_t>(ks) * 64 + (u & 63);
    kb = (n0 >> 6) + (u >> 6);
  }
}

__device__ __forceinline__ void scale_fetch(const GemmParams& p, int64_t row, int64_t kb, bool valid, ScaleSrc& d) {
  if (valid && row < p.nw && kb * 64 < p.kw) {
    const int64_t si = row * (p.kw >> 6) + kb;
    d.q = __ldg(p.qscale + si);
    d.step = __ldg(p.dq_step + (si >> 8));
    d.mean = __ldg(p.dq_mean + (si >> 8));
  } else {
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

// Decodes one unit (its 32 code bytes c0, c1 and scale inputs) into the
// 64 bf16 values of its 128-byte operand row (in registers).
__device__ __forceinline__ void decode_unit(const ScaleSrc& d, uint4 c0, uint4 c1, const float* sL, uint4 (&v)[8]) {
  const float sh = restore_scale(static_cast<int8_t>(d.q), d.step, d.mean);
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__fmul_rn(sL[2 * i], sh), __fmul_rn(sL[2 * i + 1], sh));
  const uint32_t tl0 = __byte_perm(pk[0], pk[1], 0x6420u), th0 = __byte_perm(pk[0], pk[1], 0x7531u);
  const uint32_t tl1 = __byte_perm(pk[2], pk[3], 0x6420u), th1 = __byte_perm(pk[2], pk[3], 0x7531u);
  const uint32_t tl2 = __byte_perm(pk[4], pk[5], 0x6420u), th2 = __byte_perm(pk[4], pk[5], 0x7531u);
  const uint32_t tl3 = __byte_perm(pk[6], pk[7], 0x6420u), th3 = __byte_perm(pk[6], pk[7], 0x7531u);
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int m = 0; m < 8; ++m) v[m] = decode_word(words[m], tl0, tl1, tl2, tl3, th0, th1, th2, th3);
}

// Stores a decoded unit as the 128-byte row `unit` of a swizzled operand tile.
__device__ __forceinline__ void store_unit(const uint4 (&v)[8], uint8_t* tile, int unit) {
  uint8_t* row = tile + unit * 128;
  const int sw = unit & 7;
#pragma unroll
  for (int m = 0; m < 8; ++m) *reinterpret_cast<uint4*>(row + ((m ^ sw) << 4)) = v[m];
}

// Byte offset in a code stage of byte `addr` of the unswizzled box, for a
// box written by TMA with the swizzle that matches its row pitch (32-byte
// rows: 32B swizzle, 64: 64B, 128: 128B): the 16-byte unit index is XORed
// with the address bits above 128 bytes.
template <uint32_t kPitch>
__device__ __forceinline__ uint32_t code_swz(uint32_t addr) {
  constexpr uint32_t mask = kPitch == 32 ? 1u : (kPitch == 64 ? 3u : 7u);
  return addr ^ (((addr >> 7) & mask) << 4);
}

// kF32Out: the accumulators go to outf in fp32 (no LoRA k-block; the
// dropout backward adds its masked LoRA term and rounds once).  That
// instantiation runs beside the rank-r kernel launched before it and waits
// for it before exiting, so that its completion implies that kernel's.
template <int kMode, int kC, bool kF32Out = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,       // x or dy  [m, k]
                      const __grid_constant__ CUtensorMap tm_la,      // s*u or s*v [m, rp]
                      const __grid_constant__ CUtensorMap tm_lb,      // B [nw, r] or A [r, kw]
                      const __grid_constant__ CUtensorMap tm_codes,   // codes [nw, kw/2], this CTA's share
                      const __grid_constant__ CUtensorMap tm_out,     // out [m, n] bf16, 64 x 256 boxes
                      GemmParams p) {
  using Cfg = GemmCfg<kC>;
  constexpr int S = Cfg::kStages;
  constexpr int CS = Cfg::kCStages;
  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* codes_ring = smem + Cfg::kCodeOff;
  uint64_t* afull = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* bfull = afull + S;
  uint64_t* empty = bfull + S;
  uint64_t* cfull = empty + S;
  uint64_t* cempty = cfull + CS;
  uint64_t* gdone = cempty + CS;    // [S] a decoder group's rows of the stage are written (clusters)
  uint64_t* tfull = gdone + S;
  uint64_t* tempty = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sL = reinterpret_cast<float*>(tmem_slot + 4);    // 16 floats

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&afull[i], 1);
      mbar_init(&bfull[i], Cfg::kNT + 1);
      mbar_init(&empty[i], kC);
      mbar_init(&gdone[i], Cfg::kNT);
    }
    for (int i = 0; i < CS; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], Cfg::kNT);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 16) sL[threadIdx.x] = p.lv.v[threadIdx.x];
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_la);
    tma_prefetch_desc(&tm_lb);
    tma_prefetch_desc(&tm_codes);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // every CTA of the cluster has its barriers set up before any copy or
  // commit reaches them
  if constexpr (kC > 1) cluster_sync_all();
  const uint32_t tmem_base = *tmem_slot;

  // Only the LoRA slice (bf16(s u) or bf16(s v)) is produced by the kernel
  // that precedes this one; the TMA producer waits for it before loading
  // that slice, so the main loop overlaps the predecessor's tail.
  pdl_launch_dependents();

  const int rank = kC > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int cid = kC > 1 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int ncl = kC > 1 ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
  const int nsteps = p.ksteps + p.lora_steps;
  const int ctiles = p.mc_tiles * p.n_tiles;
  const int my_tiles = ctiles > cid ? (ctiles - 1 - cid) / ncl + 1 : 0;
  const int total_its = my_tiles * nsteps;
  auto tile_m0 = [&](int t) {
    const int ct = cid + t * ncl;
    return ((ct % p.mc_tiles) * kC + rank) * kBM;
  };
  auto tile_n0 = [&](int t) {
    const int ct = cid + t * ncl;
    return (ct / p.mc_tiles) * kBN;
  };

  // Epilogue of tile t by one warp of a set of `nset` warps per TMEM lane
  // quarter (this warp is number `e` of its quarter's set): the accumulator
  // chunks of 32 columns c with c % nset == e, TMEM -> registers -> bf16 (or
  // fp32) -> global, rows of this warp's lane quarter.
  auto drain_tile = [&](int t, int e, int nset) {
    const int wq = warp & 3;
    const int m0 = tile_m0(t), n0 = tile_n0(t);
#pragma unroll 1
    for (int hc = e; hc < 2 * (kBN / 32); hc += nset) {
      const int h = hc / (kBN / 32), c = hc % (kBN / 32);
      const int64_t row = m0 + h * 128 + wq * 32 + lane;
      uint32_t v[32];
      tmem_ld32(tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + h * kBN + c * 32, v);
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
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (A)
    if (lane == 0) {
      int it = 0;
      bool waited = false, ok = true;
      for (int t = 0; t < my_tiles && ok; ++t) {
        const int m0 = tile_m0(t), n0 = tile_n0(t);
        int goff = 0;
        for (int gi = 1; gi < p.lgroups; ++gi)
          if (n0 >= p.lgstart[gi]) goff = gi * p.lgcol;
        for (int ks = 0; ks < nsteps; ++ks, ++it) {
          const int stage = it % S;
          const uint32_t phase = (it / S) & 1;
          if (!mbar_wait_cluster(&empty[stage], phase ^ 1, abort_flag, ERR_GEMM_WAIT)) { ok = false; break; }
          uint8_t* sa = smem + stage * Cfg::kStageBytes;
          uint8_t* sb = sa + Cfg::kABytes;
          if (ks < p.ksteps) {
            mbar_arrive_expect_tx(&afull[stage], Cfg::kABytes);
            tma_load_2d(&tm_a, &afull[stage], sa, ks * 64, m0);
            tma_load_2d(&tm_a, &afull[stage], sa + 16384, ks * 64, m0 + 128);
          } else {
            const int lk = (ks - p.ksteps) * 64;
            const int lka = lk + (kMode == 0 ? goff : 0);
            if (!waited) {
              pdl_wait_primary();
              waited = true;
            }
            mbar_arrive_expect_tx(&afull[stage], Cfg::kABytes + Cfg::kBBytes);
            tma_load_2d(&tm_la, &afull[stage], sa, lka, m0);
            tma_load_2d(&tm_la, &afull[stage], sa + 16384, lka, m0 + 128);
            if (kMode == 0) {
              tma_load_2d(&tm_lb, &afull[stage], sb, lk, n0);
            } else {
#pragma unroll
              for (int a = 0; a < kBN / 64; ++a) tma_load_2d(&tm_lb, &afull[stage], sb + a * 8192, n0 + 64 * a, lk);
            }
          }
        }
      }
      // Drain: the last stages' copies must land before the CTA exits, and
      // so must the commits (from every CTA of the cluster) that free them,
      // which nothing else waits for.
      const int issued = it;
      for (int j = (issued > S ? issued - S : 0); j < issued; ++j) {
        volatile int dummy = 0;
        mbar_wait(&afull[j % S], (j / S) & 1, &dummy, ERR_GEMM_WAIT);
        if (ok) mbar_wait_cluster(&empty[j % S], (j / S) & 1, &dummy, ERR_GEMM_WAIT);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kBN, kMode);
      const uint32_t lbo = (kMode == 0) ? 0u : 8192u;
      // post, for each of the first stages' phases, the bytes the other CTAs
      // of the cluster will send into it (none for the LoRA k-blocks)
      for (int j = 0; j < S && j < total_its; ++j)
        mbar_arrive_expect_tx(&bfull[j], (j % nsteps) < p.ksteps ? Cfg::kIncoming : 0u);
      int it = 0;
      for (int t = 0; t < my_tiles && !*abort_flag; ++t) {
        if (!mbar_wait(tempty, (t & 1) ^ 1, abort_flag, ERR_GEMM_WAIT)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base;
        bool ok = true;
        for (int ks = 0; ks < nsteps; ++ks, ++it) {
          const int stage = it % S;
          const uint32_t phase = (it / S) & 1;
          if (!mbar_wait(&afull[stage], phase, abort_flag, ERR_GEMM_WAIT) ||
              !mbar_wait_cluster(&bfull[stage], phase, abort_flag, ERR_GEMM_WAIT)) {
            ok = false;
            break;
          }
          if (it + S < total_its)
            mbar_arrive_expect_tx(&bfull[stage], ((it + S) % nsteps) < p.ksteps ? Cfg::kIncoming : 0u);
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
              umma_bf16_ss(d0 + h * kBN, adesc, bdesc, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if constexpr (kC > 1) umma_commit_multicast(&empty[stage], static_cast<uint16_t>((1u << kC) - 1u));
          else umma_commit(&empty[stage]);
        }
        if (!ok) break;
        umma_commit(tfull);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ TMA producer (codes)
    if (lane == 0) {
      int dit = 0;
      bool ok = true;
      for (int t = 0; t < my_tiles && ok; ++t) {
        const int n0 = tile_n0(t);
        for (int ks = 0; ks < p.ksteps; ++ks, ++dit) {
          const int cs = dit % CS;
          const uint32_t phase = (dit / CS) & 1;
          if (!mbar_wait(&cempty[cs], phase ^ 1, abort_flag, ERR_GEMM_WAIT)) { ok = false; break; }
          mbar_arrive_expect_tx(&cfull[cs], Cfg::kCBytes);
          uint8_t* dst = codes_ring + cs * Cfg::kCBytes;
          if (kMode == 0) tma_load_2d(&tm_codes, &cfull[cs], dst, ks * 32, n0 + rank * Cfg::kNU);
          else tma_load_2d(&tm_codes, &cfull[cs], dst, (n0 >> 1) + rank * static_cast<int>(Cfg::kCPitch), ks * 64);
        }
      }
      const int issued = dit;
      for (int j = (issued > CS ? issued - CS : 0); j < issued; ++j) {
        volatile int dummy = 0;
        mbar_wait(&cfull[j % CS], (j / CS) & 1, &dummy, ERR_GEMM_WAIT);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    // with several tiles, each in turn; a CTA's only tile is drained by warps
    // 4-15 together (see below)
    for (int t = 0; my_tiles > 1 && t < my_tiles; ++t) {
      if (!mbar_wait(tfull, t & 1, abort_flag, ERR_GEMM_WAIT)) break;
      tc_fence_after();
      drain_tile(t, 0, 1);
      tc_fence_before();
      mbar_arrive(tempty);
    }
  } else if (warp >= 8 && warp < 8 + Cfg::kDecoders) {
    // ------------------------------------------------------------ decoders
    constexpr int U = Cfg::kU;
    constexpr int G = Cfg::kG;
    const int dw = warp - 8;
    const int grp = dw / Cfg::kDecWarps;          // takes iterations it % G == grp
    const int wg = dw % Cfg::kDecWarps;
    const int lu0 = wg * 32 + lane;               // this thread's first local unit
    auto fetch = [&](int it, ScaleSrc (&d)[U]) {
      const bool in = it < total_its;
      const int t = in ? it / nsteps : 0;
      const int ks = in ? it % nsteps : 0;
      const int64_t n0 = tile_n0(t);
#pragma unroll
      for (int i = 0; i < U; ++i) {
        int64_t row, kb;
        unit_coords<kMode>(rank * Cfg::kNU + lu0 + 128 * i, ks, n0, row, kb);
        scale_fetch(p, row, kb, in && ks < p.ksteps, d[i]);
      }
    };
    uint8_t* const ring = smem;
    // One k-block of this group: codes from the code ring, scale inputs from
    // `sc` (loaded two own k-blocks earlier), decoded into the operand stage
    // (and sent to the other CTAs of the cluster); then `sc` is reloaded for
    // the group's k-block two turns later.  False when a wait gave up.
    auto body = [&](int it, ScaleSrc (&sc)[U]) -> bool {
      const int t = it / nsteps;
      const int ks = it % nsteps;
      const int stage = it % S;
      const uint32_t phase = (it / S) & 1;
      const bool dec = ks < p.ksteps;
      // with one unit per thread, decode into registers first: only the
      // stores wait for the stage
      uint4 dv[U][8];
      if (dec) {
        const int dit = t * p.ksteps + ks;
        const int cs = dit % CS;
        if (!mbar_wait(&cfull[cs], (dit / CS) & 1, abort_flag, ERR_GEMM_WAIT)) return false;
        const uint8_t* cb = codes_ring + cs * Cfg::kCBytes;
        uint4 cw[U][2];
#pragma unroll
        for (int i = 0; i < U; ++i) {
          const int lu = lu0 + 128 * i;
          uint32_t a0;
          if (kMode == 0) a0 = static_cast<uint32_t>(lu) * 32u;
          else a0 = static_cast<uint32_t>(lu & 63) * Cfg::kCPitch + static_cast<uint32_t>(lu >> 6) * 32u;
          constexpr uint32_t kP = kMode == 0 ? 32u : Cfg::kCPitch;
          cw[i][0] = *reinterpret_cast<const uint4*>(cb + code_swz<kP>(a0));
          cw[i][1] = *reinterpret_cast<const uint4*>(cb + code_swz<kP>(a0 + 16));
        }
        // the stage is refilled by TMA (the async proxy) once every reader released it
        fence_proxy_async_smem();
        mbar_arrive(&cempty[cs]);
        if constexpr (U == 1) decode_unit(sc[0], cw[0][0], cw[0][1], sL, dv[0]);
        else {
#pragma unroll
          for (int i = 0; i < U; ++i) dv[i][0] = cw[i][0], dv[i][1] = cw[i][1];
        }
      }
      if (!mbar_wait_cluster(&empty[stage], phase ^ 1, abort_flag, ERR_GEMM_WAIT)) return false;
      uint8_t* sb = ring + stage * Cfg::kStageBytes + Cfg::kABytes;
      if (dec) {
#pragma unroll
        for (int i = 0; i < U; ++i) {
          // two units per thread (no cluster): too many registers to decode ahead
          if constexpr (U > 1) decode_unit(sc[i], dv[i][0], dv[i][1], sL, dv[i]);
          store_unit(dv[i], sb, rank * Cfg::kNU + lu0 + 128 * i);
        }
        fence_proxy_async_smem();
      }
      if constexpr (kC > 1) {
        // the group's rows (contiguous) go to the same place in the other
        // CTAs of the cluster, in one bulk copy each, once all of them are
        // written (and fenced); gdone takes one phase per k-block, LoRA ones too
        mbar_arrive(&gdone[stage]);
        if (wg == 0 && lane == 0) {
          if (!mbar_wait(&gdone[stage], phase, abort_flag, ERR_GEMM_WAIT)) return false;
          if (dec) {
            const uint32_t src = smem_u32(sb) + static_cast<uint32_t>(rank * Cfg::kNU) * 128u;
            const uint32_t bar = smem_u32(&bfull[stage]);
#pragma unroll
            for (int q = 1; q < kC; ++q) {
              const uint32_t peer = static_cast<uint32_t>((rank + q) % kC);
              bulk_copy_s2cluster(map_to_rank(src, peer), src, Cfg::kNU * 128u, map_to_rank(bar, peer));
            }
          }
        }
      }
      mbar_arrive(&bfull[stage]);
      fetch(it + 2 * G, sc);
      return true;
    };
    ScaleSrc sa[U], sb2[U];
    fetch(grp, sa);
    fetch(grp + G, sb2);
    for (int it = grp; it < total_its; it += 2 * G) {
      if (!body(it, sa)) break;
      if (it + G < total_its && !body(it + G, sb2)) break;
    }
  }

  // A CTA with one tile: warps 4-15 (the decoders are done by now) drain its
  // accumulators together, three warps per TMEM lane quarter.  (With more
  // tiles a decoder could reach tfull while it is still two tiles behind,
  // which its parity wait could not tell apart; then warps 4-7 drain alone.)
  // The bf16 tile goes through shared memory (the operand stages, free once
  // the last MMA has completed): each warp writes its TMEM chunks as bf16
  // into four 64-column boxes of [256 rows][128 B] (128-byte swizzle), and
  // one thread stores the boxes with TMA, so that the writes to global memory
  // are whole lines rather than a lane's 16 bytes of each of 32 rows.
  if (warp >= 4 && my_tiles == 1) {
    if (mbar_wait(tfull, 0, abort_flag, ERR_GEMM_WAIT)) {
      tc_fence_after();
      if constexpr (kF32Out) {
        drain_tile(0, (warp - 4) >> 2, 3);
      } else {
        const int wq = warp & 3, e = (warp - 4) >> 2;
        const uint32_t st0 = smem_u32(smem);
#pragma unroll 1
        for (int hc = e; hc < 2 * (kBN / 32); hc += 3) {
          const int h = hc / (kBN / 32), c = hc % (kBN / 32);
          const uint32_t row = static_cast<uint32_t>(h * 128 + wq * 32 + lane);
          uint32_t v[32];
          tmem_ld32(tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + h * kBN + c * 32, v);
          tmem_ld_wait();
          const uint32_t box = st0 + static_cast<uint32_t>(c >> 1) * 32768u + row * 128u;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t j = static_cast<uint32_t>((c & 1) * 4 + k);
            const uint32_t a = box + ((j ^ (row & 7u)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                         "r"(pack_bf16x2(__uint_as_float(v[8 * k + 0]), __uint_as_float(v[8 * k + 1]))),
                         "r"(pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3]))),
                         "r"(pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5]))),
                         "r"(pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7])))
                         : "memory");
          }
        }
      }
    }
    if constexpr (!kF32Out) {
      fence_proxy_async_smem();
      named_bar_sync(1, 384);       // warps 4-15
      if (warp == 4 && lane == 0 && !*abort_flag) {
        const int m0 = tile_m0(0), n0 = tile_n0(0);
        for (int b = 0; b < kBN / 64; ++b)
          if (n0 + 64 * b < p.n) tma_store_2d(&tm_out, smem + b * 32768, n0 + 64 * b, m0);
        bulk_commit_group();
        bulk_wait_group0();
      }
    }
  }
  if constexpr (kF32Out) {
    if (threadIdx.x == 0) pdl_wait_primary();
  }
  __syncwarp();
  __syncthreads();
  if constexpr (kC > 1) {
    // no CTA leaves while another may still copy into its shared memory;
    // after a wait gave up, copies already issued are given time to land
    cluster_sync_all();
    if (*abort_flag) {
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < 100000ull) {
      }
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace qn
