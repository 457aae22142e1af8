// qlora_nf4.cu -- the C ABI of libqlora_nf4.so (declared in include/qlora_nf4.h).
//
// Host side only: argument checks, the workspace plan, tensor-map encoding
// and kernel launches.  Every launch after the first of a call uses
// programmatic stream serialization, so a kernel's prologue overlaps the
// tail of its predecessor; each kernel waits for its predecessor
// (griddepcontrol.wait) before touching global memory.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <cstdio>
#include <array>
#include <cstdlib>
#include <mutex>
#include <utility>

#include "../../include/qlora_nf4.h"
#include "adamw8.cuh"
#include "common.cuh"
#include "dropout.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "lora_small.cuh"
#include "merge.cuh"
#include "nf4_storage.cuh"

using namespace qn;

namespace {

// ------------------------------------------------------------------ levels

// The 16 NF4 levels [QLoRA glossary, NF4 snippet]: standard-normal quantiles
// at the first 8 of 9 evenly spaced probabilities from 0.9677083 to 0.5
// (positive side) and the negated quantiles at the first 7 of 8 (negative
// side), an exact zero, sorted, divided by the largest; computed in fp64
// and rounded once to fp32.  The inverse CDF is found by bisection on
// Phi(x) = erfc(-x / sqrt 2) / 2.
double phi(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double phi_inverse(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 400 && hi - lo > 0.0; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (phi(mid) < p) lo = mid;
    else hi = mid;
  }
  return 0.5 * (lo + hi);
}

Levels compute_levels() {
  const double start = 0.9677083, stop = 0.5;
  double v[16];
  int n = 0;
  {
    const double step = (stop - start) / 7.0;           // 8 points, drop the last
    for (int i = 0; i < 7; ++i) v[n++] = -phi_inverse(static_cast<double>(i) * step + start);
  }
  v[n++] = 0.0;
  {
    const double step = (stop - start) / 8.0;           // 9 points, drop the last
    for (int i = 0; i < 8; ++i) v[n++] = phi_inverse(static_cast<double>(i) * step + start);
  }
  // sort ascending (insertion sort on 16 values)
  for (int i = 1; i < 16; ++i)
    for (int j = i; j > 0 && v[j - 1] > v[j]; --j) {
      const double t = v[j];
      v[j] = v[j - 1];
      v[j - 1] = t;
    }
  const double top = v[15];
  Levels L;
  for (int i = 0; i < 16; ++i) L.v[i] = static_cast<float>(v[i] / top);
  return L;
}

const Levels& levels() {
  static const Levels L = compute_levels();
  return L;
}

// bf16 bits of a finite float, rounded to nearest even.
uint16_t bf16_bits_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// The decode GEMV's lookup table: code byte e -> (bf16(level[e & 15]) in
// the low half, bf16(level[e >> 4]) in the high half).
const uint32_t* gemv_lut() {
  static const std::array<uint32_t, 256> T = [] {
    std::array<uint32_t, 256> t{};
    const Levels& L = levels();
    for (int e = 0; e < 256; ++e)
      t[e] = bf16_bits_rne(L.v[e & 15]) | (static_cast<uint32_t>(bf16_bits_rne(L.v[e >> 4])) << 16);
    return t;
  }();
  return T.data();
}

// ------------------------------------------------------------------ device info

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

bool device_is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

// ------------------------------------------------------------------ launches

// Launches `kernel`; `pdl` lets it start while its predecessor in the stream
// (always a kernel of this library within the same call) finishes, and
// `cluster` > 1 groups consecutive CTAs into thread-block clusters.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      bool pdl, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = n ? attr : nullptr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   bool pdl, Args&&... args) {
  return launch_ex(kernel, grid, block, smem, st, pdl, 1, std::forward<Args>(args)...);
}

template <typename K>
bool set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes)) == cudaSuccess;
}

// ------------------------------------------------------------------ tensor maps

// The CUDA error behind the last QN_ERR_CUDA of this host thread, and an
// optional detail (which step failed) reported with it.
thread_local cudaError_t t_last_error = cudaSuccess;
thread_local char t_last_detail[160] = "";

void set_detail(const char* what, int code) {
  std::snprintf(t_last_detail, sizeof(t_last_detail), "%s (driver result %d)", what, code);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 row-major [outer, inner] with a row stride of `ld` elements; box
// {box_inner, box_outer}; 128-byte swizzle; zero fill out of bounds.
bool tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
               uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ checks

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

qn_status check_weight(const qn_nf4_weight* w) {
  if (!w || !w->codes || !w->qscale || !w->dq_step || !w->dq_mean) return QN_ERR_ARG;
  if (w->n_out <= 0 || w->k_in <= 0 || (w->k_in % 64) != 0) return QN_ERR_SHAPE;
  if (!aligned16(w->codes) || !aligned16(w->qscale) || !aligned16(w->dq_step) ||
      !aligned16(w->dq_mean))
    return QN_ERR_ALIGN;
  return QN_OK;
}

qn_status check_layer(const qn_nf4_weight* w, int r) {
  qn_status s = check_weight(w);
  if (s != QN_OK) return s;
  if ((w->n_out % 64) != 0) return QN_ERR_SHAPE;
  if (r < 0 || r > kMaxRank || (r % 8) != 0) return QN_ERR_SHAPE;
  if (w->n_out > (int64_t{1} << 31) || w->k_in > (int64_t{1} << 31)) return QN_ERR_SHAPE;
  return QN_OK;
}

// ------------------------------------------------------------------ small-product plans

// Workspace layout (all offsets 256-byte aligned):
//   scaled  bf16 [m, rp]   bf16(s u) (forward) / bf16(s v) (backward)
//   uplain  bf16 [m, r]    u recomputed in the backward
//   vplain  bf16 [m, r]    v = dy B
//   dxf     fp32 [m, k_in]  dy W_hat before the dropout LoRA term (dropout calls only)
//   sync    2 x uint32     the decode call's counters (zero between calls)
struct Layout {
  size_t scaled, uplain, vplain, dxf, sync, total;
};

struct GemvPlan {
  int nh;          // 1: up to 8 tokens, 2: up to 16
  int grid;        // CTAs
  int rg_batch;    // 16-row units whose partial tiles fit in shared memory at once
  size_t smem;
};

// false when even one 16-row unit's partial tiles do not fit (K too large).
template <int NH>
bool plan_gemv_nh(int64_t t, int64_t n, int64_t k, int r, GemvPlan* g) {
  const int64_t nru = n / 16, nkr = k / 256;
  // u = x A^T takes one CTA per 8 rank rows, beside the GEMV
  const int avail = std::max(1, sm_count() - r / 8);
  g->grid = static_cast<int>(std::min<int64_t>(avail, nru));
  const int64_t ruc = ceil_div(nru, g->grid);
  const int64_t fixed = gemv_smem_layout<NH>(kGemvHostBase, static_cast<int>(nkr), 0, static_cast<int>(t)).total;
  const int64_t per_ru = gemv_smem_layout<NH>(kGemvHostBase, static_cast<int>(nkr), 1, static_cast<int>(t)).total - fixed;
  const int64_t fit = (kGemvSmemBudget - fixed) / per_ru;
  if (fit < 1) return false;
  g->rg_batch = static_cast<int>(std::min(ruc, fit));
  while (g->rg_batch > 1 &&
         gemv_smem_layout<NH>(kGemvHostBase, static_cast<int>(nkr), g->rg_batch, static_cast<int>(t)).total > kGemvSmemBudget)
    --g->rg_batch;
  g->smem = gemv_smem_layout<NH>(kGemvHostBase, static_cast<int>(nkr), g->rg_batch, static_cast<int>(t)).total;
  return g->smem <= static_cast<size_t>(kGemvSmemBudget);
}

bool plan_gemv(int64_t t, int64_t n, int64_t k, int r, GemvPlan* g) {
  g->nh = (t <= 8) ? 1 : 2;
  return g->nh == 1 ? plan_gemv_nh<1>(t, n, k, r, g) : plan_gemv_nh<2>(t, n, k, r, g);
}

Layout layout(int64_t m, int64_t n, int64_t k, int r, bool dropout = false) {
  Layout L;
  const int64_t rp = round_up(r, 64);
  size_t off = 0;
  L.scaled = off;  off = align256(off + static_cast<size_t>(m) * rp * 2);
  L.uplain = off;  off = align256(off + static_cast<size_t>(m) * r * 2);
  L.vplain = off;  off = align256(off + static_cast<size_t>(m) * r * 2);
  L.dxf = off;     off = align256(off + (dropout ? static_cast<size_t>(m) * k * 4 : 0));
  L.sync = off;    off += 256;
  L.total = off;
  return L;
}

SmallProblem small_problem(int kind, const void* X, const void* W, int w_transposed, int64_t rows,
                           int64_t red, int r, float s) {
  SmallProblem p = {};
  p.kind = kind;
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.W = static_cast<const __nv_bfloat16*>(W);
  p.w_transposed = w_transposed;
  p.rows = rows;
  p.red = red;
  p.r = r;
  p.s = s;
  p.tiles = static_cast<int>(ceil_div(rows, kSmallTile));
  // few row tiles (decode shapes): split the rank columns in groups of 16
  p.csplit = (p.tiles < 8 && r % 16 == 0 && r > 16) ? r / 16 : 1;
  p.rj = r / p.csplit;

  p.rp = static_cast<int>(round_up(r, 64));
  p.pad = p.rp - r;
  p.ldp = r;
  p.ldx = kind == 0 ? red : rows;
  p.ldw = (kind == 0 && !w_transposed) ? red : r;
  return p;
}

// lora_rank_kernel<NT> for NT = 1..16 (8 to 128 rank columns per tile).
struct RankKernels {
  typedef void (*Fn)(const SmallMaps, SmallBatch);
  Fn fn[17] = {};
  bool ok = true;
  template <int NT>
  void add() {
    fn[NT] = lora_rank_kernel<NT>;
    ok = ok && set_smem(lora_rank_kernel<NT>, rank_smem_bytes(kRankMaxStages, 2));
  }
  template <int... NTs>
  void add_all(std::integer_sequence<int, NTs...>) {
    (add<NTs + 1>(), ...);
  }
  RankKernels() { add_all(std::make_integer_sequence<int, 16>{}); }
};

const RankKernels& rank_kernels() {
  static const RankKernels k;
  return k;
}

// Launches one or two rank-r products as one kernel: one thread-block
// cluster per tile, whose CTAs split the reduction and combine over
// distributed shared memory.  Every operand is read through a tensor map of
// 64 x 64 boxes: x / dy along their rows, the rank-side operand with zero
// fill past rank r.  max_ctas > 0 caps the CTAs (the kernel then leaves
// the other SMs to a kernel running beside it).  side: exactly max_ctas CTAs
// with a deep ring, one per SM (their shared memory does not fit twice), each
// reducing whole tiles, to run beside a GEMM on the SMs it leaves idle.
cudaError_t run_small(SmallProblem* probs, int count, cudaStream_t st, bool pdl, int max_ctas = 0,
                      bool side = false) {
  SmallBatch b = {};
  if (count < 1 || count > kSmallMaxProblems) return cudaErrorInvalidValue;
  // one launch has one tile width: its problems share the rank
  for (int i = 1; i < count; ++i)
    if (probs[i].r != probs[0].r) return cudaErrorInvalidValue;
  b.count = count;
  // one launch has one tile width: problems that disagree keep all columns
  for (int i = 0; i < count; ++i) {
    if (probs[i].rj != probs[0].rj || max_ctas > 0) {
      for (int k = 0; k < count; ++k) {
        probs[k].csplit = 1;
        probs[k].rj = probs[k].r;
      }
      break;
    }
  }
  int64_t clusters = 0;
  int rj = 0;
  for (int i = 0; i < count; ++i) {
    clusters += static_cast<int64_t>(probs[i].tiles) * probs[i].csplit;
    rj = std::max(rj, probs[i].rj);
  }
  const RankKernels& K = rank_kernels();
  const int nt = rj / 8;
  if (!K.ok || nt < 1 || nt > 16 || clusters < 1) return cudaErrorInvalidValue;
  b.wboxes = rj > 64 ? 2 : 1;
  b.stages = side ? kRankMaxStages : (b.wboxes == 1 ? 6 : 4);   // side: one CTA per SM, else two
  const size_t smem = rank_smem_bytes(b.stages, b.wboxes);
  int64_t slots = 2 * static_cast<int64_t>(sm_count());
  if (max_ctas > 0) slots = std::min<int64_t>(slots, max_ctas);
  // CTAs per cluster: as many as keep every cluster resident at once
  int cs = 1;
  for (int i = 0; i < count && !side; ++i) {
    int64_t c = std::min<int64_t>(slots / clusters, kMaxCluster);
    c = std::min<int64_t>(c, ceil_div(probs[i].red, 64));
    cs = std::max<int>(cs, static_cast<int>(std::max<int64_t>(c, 1)));
  }
  SmallMaps maps;
  bool ok = true;
  for (int i = 0; i < count; ++i) {
    SmallProblem& P = probs[i];
    P.chunk = round_up(ceil_div(P.red, cs), 64);
    if (P.kind == 0) {
      ok = ok && tmap_bf16(&maps.x[i], P.X, P.red, P.rows, P.ldx, 64, 64);
      if (!P.w_transposed) ok = ok && tmap_bf16(&maps.w[i], P.W, P.red, P.r, P.ldw, 64, 64);
      else ok = ok && tmap_bf16(&maps.w[i], P.W, P.r, P.red, P.ldw, 64, 64);
    } else {
      ok = ok && tmap_bf16(&maps.x[i], P.X, P.rows, P.red, P.ldx, 64, 64);
      ok = ok && tmap_bf16(&maps.w[i], P.W, P.r, P.red, P.ldw, 64, 64);
    }
    b.p[i] = P;
    b.cend[i] = (i ? b.cend[i - 1] : 0) + P.tiles * P.csplit;
  }
  if (!ok) return cudaErrorInvalidValue;
  for (int i = count; i < kSmallMaxProblems; ++i) {
    maps.x[i] = maps.x[0];
    maps.w[i] = maps.w[0];
  }
  b.clusters = static_cast<int>(clusters);
  b.cs = cs;
  const int64_t grid_clusters = std::min<int64_t>(clusters, std::max<int64_t>(slots / cs, 1));
  return launch_ex(K.fn[nt], dim3(static_cast<unsigned>(grid_clusters * cs)), dim3(kRankThreads), smem, st,
                   pdl, cs, maps, b);
}

// Runs `count` problems, as few launches as the rule of one rank per launch
// and kSmallMaxProblems per launch allow (order kept within a rank).
cudaError_t run_small_by_rank(SmallProblem* probs, int count, cudaStream_t st, bool pdl, int side_ctas) {
  bool done[2 * kSmallMaxProblems + 2] = {};
  bool first = true;
  for (int i = 0; i < count; ++i) {
    if (done[i]) continue;
    SmallProblem batch[kSmallMaxProblems];
    int c = 0;
    for (int j = i; j < count && c < kSmallMaxProblems; ++j)
      if (!done[j] && probs[j].r == probs[i].r) {
        batch[c++] = probs[j];
        done[j] = true;
      }
    const cudaError_t e = side_ctas > 0 ? run_small(batch, c, st, pdl && first, side_ctas, true)
                                        : run_small(batch, c, st, pdl && first);
    if (e != cudaSuccess) return e;
    first = false;
  }
  return cudaSuccess;
}

// s = fl32(alpha / r): one IEEE single division on the host.
float lora_scale(float alpha, int r) { return r > 0 ? alpha / static_cast<float>(r) : 0.f; }

// ------------------------------------------------------------------ GEMM launch

// Codes [n_out, k_in/2] bytes read in boxes of `inner` bytes x `rows` rows,
// with the swizzle whose span matches the box's row (32, 64 or 128 bytes).
bool tmap_codes(CUtensorMap* m, const qn_nf4_weight* w, uint32_t inner, uint32_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(w->k_in / 2), static_cast<cuuint64_t>(w->n_out)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(w->k_in / 2)};
  const cuuint32_t box[2] = {inner, rows};
  const cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw = inner == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                : inner == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w->codes, dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) set_detail("tensor map of the codes (GEMM)", static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

// One instantiation of the fused GEMM: its shared-memory attribute, set
// once, and how many of its clusters fit on the device at once.
template <int kMode, int kC, bool kF32Out>
struct GemmKernel {
  bool ok = false;
  int max_clusters = 0;
  GemmKernel() {
    auto fn = qlora_gemm_kernel<kMode, kC, kF32Out>;
    ok = set_smem(fn, GemmCfg<kC>::kSmemBytes);
    if (!ok) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(kC));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = GemmCfg<kC>::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = sm_count() / kC;
    }
    max_clusters = n;
  }
  static const GemmKernel& get() {
    static const GemmKernel k;
    return k;
  }
};

// CTAs per cluster for an M x N problem: of 2, 4 and 1 (in that order of
// preference: pairs share the decode with the least lock-step between CTAs),
// one that divides the M-tiles and needs no more waves of resident clusters
// than any other.
int forced_cluster() {
  static const int v = [] {
    const char* e = std::getenv("QN_GEMM_CLUSTER");
    const int c = e ? std::atoi(e) : 0;
    return (c == 1 || c == 2 || c == 4) ? c : 0;
  }();
  return v;
}

template <int kMode, bool kF32Out>
int gemm_cluster(int64_t m_tiles, int64_t n_tiles) {
  const int f = forced_cluster();
  if (f && m_tiles % f == 0) return f;
  const int cand[3] = {2, 4, 1};
  const int maxc[3] = {GemmKernel<kMode, 2, kF32Out>::get().max_clusters,
                       GemmKernel<kMode, 4, kF32Out>::get().max_clusters,
                       GemmKernel<kMode, 1, kF32Out>::get().max_clusters};
  int best = 1;
  int64_t best_waves = -1;
  for (int i = 0; i < 3; ++i) {
    const int c = cand[i];
    if (m_tiles % c != 0 || maxc[i] <= 0) continue;
    const int64_t waves = ceil_div(m_tiles / c * n_tiles, maxc[i]);
    if (best_waves < 0 || waves < best_waves) {
      best = c;
      best_waves = waves;
    }
  }
  return best;
}

struct GemmPlan {
  int c;          // CTAs per cluster
  int grid;       // CTAs launched
};

template <int kMode, bool kF32Out>
GemmPlan plan_gemm(int64_t m, int64_t n) {
  const int64_t m_tiles = ceil_div(m, kBM), n_tiles = ceil_div(n, kBN);
  GemmPlan g;
  g.c = gemm_cluster<kMode, kF32Out>(m_tiles, n_tiles);
  const int maxc = g.c == 4 ? GemmKernel<kMode, 4, kF32Out>::get().max_clusters
                   : g.c == 2 ? GemmKernel<kMode, 2, kF32Out>::get().max_clusters
                              : GemmKernel<kMode, 1, kF32Out>::get().max_clusters;
  const int64_t ctiles = m_tiles / g.c * n_tiles;
  g.grid = static_cast<int>(std::min<int64_t>(ctiles, std::max(maxc, 1)) * g.c);
  return g;
}

template <int kMode, int kC, bool kF32Out>
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tla, const CUtensorMap& tlb,
                        const CUtensorMap& tout, const qn_nf4_weight* w, GemmParams& p, int grid, cudaStream_t st,
                        bool pdl) {
  if (!GemmKernel<kMode, kC, kF32Out>::get().ok) return cudaErrorInvalidValue;
  CUtensorMap tc;
  const bool ok = kMode == 0 ? tmap_codes(&tc, w, 32, GemmCfg<kC>::kNU)
                             : tmap_codes(&tc, w, GemmCfg<kC>::kCPitch, 64);
  if (!ok) return cudaErrorInvalidValue;
  p.mc_tiles = p.m_tiles / kC;
  return launch_ex(qlora_gemm_kernel<kMode, kC, kF32Out>, dim3(static_cast<unsigned>(grid)), dim3(kGemmThreads),
                   GemmCfg<kC>::kSmemBytes, st, pdl, kC, ta, tla, tlb, tc, tout, p);
}

// LoRA groups of a sibling forward: group i's output rows start at start[i]
// (multiples of the 256-row tile) and its LoRA block is columns
// i * col .. of s*u, a buffer `width` columns wide.
constexpr int kMaxSiblingGroups = 4;

struct LoraGroups {
  int count = 1;
  int64_t start[4] = {0, 0, 0, 0};
  int col = 0;
  int64_t width = 0;
};

template <int kMode, bool kF32Out = false>
cudaError_t run_gemm(const void* a, const void* la, const void* lb, const qn_nf4_weight* w,
                     int64_t m, int r, void* out, cudaStream_t st, bool pdl, float* outf = nullptr,
                     const LoraGroups& lg = LoraGroups()) {
  GemmParams p = {};
  p.codes = w->codes;
  p.qscale = w->qscale;
  p.dq_step = w->dq_step;
  p.dq_mean = w->dq_mean;
  p.nw = w->n_out;
  p.kw = w->k_in;
  p.m = m;
  p.n = kMode == 0 ? w->n_out : w->k_in;
  p.k = kMode == 0 ? w->k_in : w->n_out;
  p.ksteps = static_cast<int>(p.k / 64);
  const int64_t rp = round_up(r, 64);
  p.lora_steps = static_cast<int>(rp / 64);
  p.m_tiles = static_cast<int>(ceil_div(m, kBM));
  p.n_tiles = static_cast<int>(ceil_div(p.n, kBN));
  p.out = static_cast<__nv_bfloat16*>(out);
  p.outf = outf;
  p.lv = levels();
  p.lgroups = lg.count;
  p.lgcol = lg.col;
  for (int i = 0; i < 4; ++i) p.lgstart[i] = lg.start[i];
  const int64_t law = lg.count > 1 ? lg.width : rp;
  CUtensorMap ta, tla, tlb;
  if (!tmap_bf16(&ta, a, p.k, m, p.k, 64, 128)) return cudaErrorInvalidValue;
  if (r > 0) {
    if (!tmap_bf16(&tla, la, law, m, law, 64, 128)) return cudaErrorInvalidValue;
    if (kMode == 0) {
      if (!tmap_bf16(&tlb, lb, r, w->n_out, r, 64, kBN)) return cudaErrorInvalidValue;
    } else {
      if (!tmap_bf16(&tlb, lb, w->k_in, r, w->k_in, 64, 64)) return cudaErrorInvalidValue;
    }
  } else {
    tla = ta;
    tlb = ta;
  }
  // bf16 output: 64-column x 256-row boxes for the TMA stores of the epilogue
  CUtensorMap tout = ta;
  if (!kF32Out && !tmap_bf16(&tout, out, p.n, m, p.n, 64, 256)) return cudaErrorInvalidValue;
  const GemmPlan g = plan_gemm<kMode, kF32Out>(m, p.n);
  switch (g.c) {
    case 4: return launch_gemm<kMode, 4, kF32Out>(ta, tla, tlb, tout, w, p, g.grid, st, pdl);
    case 2: return launch_gemm<kMode, 2, kF32Out>(ta, tla, tlb, tout, w, p, g.grid, st, pdl);
    default: return launch_gemm<kMode, 1, kF32Out>(ta, tla, tlb, tout, w, p, g.grid, st, pdl);
  }
}

template <int NH>
cudaError_t run_gemv_kernel(const CUtensorMap& tm, const GemvParams& p, int grid, size_t smem, cudaStream_t st,
                            bool pdl) {
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, [] { ok = set_smem(qlora_gemv_kernel<NH>, kGemvSmemBudget); });
  if (!ok || smem > static_cast<size_t>(kGemvSmemBudget)) return cudaErrorInvalidValue;
  return launch(qlora_gemv_kernel<NH>, dim3(grid), dim3(GemvCfg<NH>::kThreads), smem, st, pdl, tm, p);
}


// First-level encode: 4 blocks per warp per pass, kEncodeUnroll passes of
// loads in flight, at most 8 CTAs of 8 warps per SM.
constexpr int kEncodeUnroll = 4;
cudaError_t run_encode(const void* w_bf16, const qn_nf4_weight* out, float* absmax, int64_t nblk, cudaStream_t st) {
  int64_t grid = ceil_div(nblk, 4 * kEncodeUnroll * 8);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (grid > cap) grid = cap;
  return launch(nf4_encode_kernel<kEncodeUnroll>, dim3(static_cast<unsigned>(std::max<int64_t>(grid, 1))), dim3(256),
                0, st, false, static_cast<const uint4*>(w_bf16), reinterpret_cast<uint32_t*>(out->codes), absmax,
                nblk, levels());
}

qn_status to_status(cudaError_t e) {
  if (e == cudaSuccess) return QN_OK;
  t_last_error = e;
  return QN_ERR_CUDA;
}

// Clears the detail at the start of a call, so that a later failure with no
// detail does not report an old one.
void clear_detail() { t_last_detail[0] = 0; }

// SMs a fused GEMM of m x n leaves idle (its CTAs take one tile each when
// there are fewer tiles than SMs); 0 when too few to be worth a side kernel.
constexpr int kMinSideSMs = 8;
template <int kMode, bool kF32Out = false>
int side_sms(int64_t m, int64_t n) {
  const int64_t spare = sm_count() - plan_gemm<kMode, kF32Out>(m, n).grid;
  return spare >= kMinSideSMs ? static_cast<int>(spare) : 0;
}

// Forward pieces shared by both paths: u = x A^T -> u_save, bf16(s u).
cudaError_t run_lora_down_fwd(const void* x, int64_t m, const qn_nf4_weight* w, const void* A, int r,
                              float s, void* u_save, const Layout& L, uint8_t* ws, cudaStream_t st,
                              bool pdl, int max_ctas = 0, bool side = false) {
  SmallProblem pu = small_problem(0, x, A, 0, m, w->k_in, r, s);
  pu.plain = static_cast<__nv_bfloat16*>(u_save);
  pu.scaled = reinterpret_cast<__nv_bfloat16*>(ws + L.scaled);
  return run_small(&pu, 1, st, pdl, max_ctas, side);
}

qn_status validate_fwd(const void* x, int64_t m, const qn_nf4_weight* w, const void* A, const void* B,
                       int r, float alpha, const void* y, const void* u_save, const void* ws,
                       size_t ws_bytes, bool dropout = false) {
  qn_status s = check_layer(w, r);
  if (s != QN_OK) return s;
  if (m < 0) return QN_ERR_SHAPE;
  if (m == 0) return QN_OK;
  if (!x || !y) return QN_ERR_ARG;
  if (r > 0 && (!A || !B || !std::isfinite(alpha))) return QN_ERR_ARG;
  if (!aligned16(x) || !aligned16(y) || (r > 0 && (!aligned16(A) || !aligned16(B))) ||
      (u_save && !aligned16(u_save)))
    return QN_ERR_ALIGN;
  const Layout L = layout(m, w->n_out, w->k_in, r, dropout);
  if (!ws || ws_bytes < L.total) return QN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  return QN_OK;
}

// ------------------------------------------------------------------ failure-detection self-test

// Bit of the device error word set by the self-test below.
constexpr unsigned int kErrSelftestWait = QN_WAIT_SELFTEST;

// One thread waits on an mbarrier phase that nothing completes, with the
// same bounded wait as every pipeline of the library: it gives up after the
// wait limit, sets its bit in the device error word and the kernel returns.
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, kErrSelftestWait);
}

// ------------------------------------------------------------------ dropout

bool dropout_rate_ok(float p) { return std::isfinite(p) && p >= 0.f && p < 1.f; }

// floor(p * 2^32): a Philox word below it drops its element.  p * 2^32 is
// exact in double for an fp32 p.
uint32_t dropout_threshold(float p) {
  return static_cast<uint32_t>(std::floor(static_cast<double>(p) * 4294967296.0));
}

// s_d = s / (1 - p), one rounding to fp32 (1 - p is exact in double).
float dropout_scale(float s, float p) {
  return static_cast<float>(static_cast<double>(s) / (1.0 - static_cast<double>(p)));
}

cudaError_t run_dropout(const void* x, int64_t m, int64_t k, float p, uint64_t seed, uint64_t offset,
                        void* x_drop, uint32_t* keep, cudaStream_t st) {
  DropoutParams d = {};
  d.x = static_cast<const uint4*>(x);
  d.xm = static_cast<uint4*>(x_drop);
  d.keep = keep;
  d.n8 = m * k / 8;
  d.key0 = static_cast<uint32_t>(seed);
  d.key1 = static_cast<uint32_t>(seed >> 32);
  d.off0 = static_cast<uint32_t>(offset);
  d.off1 = static_cast<uint32_t>(offset >> 32);
  d.thresh = dropout_threshold(p);
  const int64_t chunks = ceil_div(d.n8, 128);
  const int64_t blocks = std::min<int64_t>(ceil_div(chunks, kDropoutThreads / 32), int64_t{8} * sm_count());
  return launch(lora_dropout_kernel, dim3(static_cast<unsigned>(std::max<int64_t>(blocks, 1))),
                dim3(kDropoutThreads), 0, st, false, d);
}

cudaError_t run_dx_dropout(const float* base, const uint32_t* keep, const void* v, const void* A, void* dx,
                           int64_t m, int64_t k, int r, float sd, cudaStream_t st) {
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, [] { ok = set_smem(lora_dx_dropout_kernel, dx_dropout_smem_bytes(kMaxRank)); });
  if (!ok) return cudaErrorInvalidValue;
  DxDropoutParams d = {};
  d.base = base;
  d.keep = keep;
  d.v = static_cast<const __nv_bfloat16*>(v);
  d.A = static_cast<const __nv_bfloat16*>(A);
  d.dx = static_cast<__nv_bfloat16*>(dx);
  d.M = m;
  d.K = k;
  d.r = r;
  d.sd = sd;
  // persistent CTAs: as many as fit at once, each walking tiles of 64 x 128
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lora_dx_dropout_kernel, kDxThreads,
                                                    dx_dropout_smem_bytes(r)) != cudaSuccess || per_sm < 1)
    return cudaErrorInvalidValue;
  const int64_t tiles = ceil_div(m, kDxRows) * ceil_div(k, kDxCols);
  const int64_t grid = std::min<int64_t>(tiles, static_cast<int64_t>(per_sm) * sm_count());
  return launch(lora_dx_dropout_kernel, dim3(static_cast<unsigned>(std::max<int64_t>(grid, 1))), dim3(kDxThreads),
                dx_dropout_smem_bytes(r), st, true, d);
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

int qn_abi_version(void) { return QN_ABI_VERSION; }

const char* qn_last_error_string(void) {
  if (t_last_error == cudaSuccess) return "no error";
  if (t_last_detail[0]) return t_last_detail;
  return cudaGetErrorString(t_last_error);
}

const char* qn_status_string(qn_status s) {
  switch (s) {
    case QN_OK: return "ok";
    case QN_ERR_ARG: return "invalid argument";
    case QN_ERR_SHAPE: return "unsupported shape";
    case QN_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QN_ERR_WORKSPACE: return "workspace missing or too small";
    case QN_ERR_CUDA: return "CUDA error";
    case QN_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case QN_ERR_UNSUPPORTED: return "device is not sm_100";
  }
  return "unknown status";
}

void nf4_levels(float out[16]) {
  if (!out) return;
  const Levels& L = levels();
  for (int i = 0; i < 16; ++i) out[i] = L.v[i];
}

qn_status qn_device_error(int* flags_out) {
  if (!flags_out) return QN_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return QN_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) return QN_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return QN_ERR_CUDA;
  *flags_out = static_cast<int>(v);
  return QN_OK;
}

qn_status qn_selftest_bounded_wait(qn_stream_t stream) {
  clear_detail();
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  return to_status(launch(selftest_wait_kernel, dim3(1), dim3(32), 0, reinterpret_cast<cudaStream_t>(stream), false));
}

size_t nf4_quantize_workspace_bytes(int64_t n_out, int64_t k_in) {
  if (n_out <= 0 || k_in <= 0) return 0;
  return align256(static_cast<size_t>(n_out) * (k_in / 64) * sizeof(float));
}

qn_status nf4_quantize(const void* w_bf16, const qn_nf4_weight* out, void* ws, size_t ws_bytes,
                       qn_stream_t stream) {
  clear_detail();
  qn_status s = check_weight(out);
  if (s != QN_OK) return s;
  if (!w_bf16) return QN_ERR_ARG;
  if (!aligned16(w_bf16)) return QN_ERR_ALIGN;
  if (!ws || ws_bytes < nf4_quantize_workspace_bytes(out->n_out, out->k_in)) return QN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nblk = out->n_out * (out->k_in / 64);
  const int64_t ngroups = ceil_div(nblk, 256);
  float* absmax = static_cast<float*>(ws);
  cudaError_t e = run_encode(w_bf16, out, absmax, nblk, st);
  if (e != cudaSuccess) return to_status(e);
  e = launch(nf4_dq_kernel, dim3(static_cast<unsigned>(ceil_div(ngroups, 8))), dim3(256), 0, st, false,
             static_cast<const float*>(absmax), nblk, out->qscale, out->dq_step, out->dq_mean, ngroups);
  return to_status(e);
}

qn_status nf4_dequantize(const qn_nf4_weight* w, void* w_hat_bf16, qn_stream_t stream) {
  clear_detail();
  qn_status s = check_weight(w);
  if (s != QN_OK) return s;
  if (!w_hat_bf16) return QN_ERR_ARG;
  if (!aligned16(w_hat_bf16)) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n8 = w->n_out * w->k_in / 8;
  constexpr int kU = 4;
  int64_t grid = ceil_div(n8, 256 * kU);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (grid > cap) grid = cap;
  return to_status(launch(nf4_dequant_kernel<kU>, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, false,
                          reinterpret_cast<const uint32_t*>(w->codes), static_cast<const int8_t*>(w->qscale),
                          static_cast<const float*>(w->dq_step), static_cast<const float*>(w->dq_mean),
                          static_cast<uint4*>(w_hat_bf16), n8, levels()));
}

size_t qlora_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int r) {
  if (m < 0 || n_out <= 0 || k_in <= 0 || r < 0) return 0;
  return layout(m, n_out, k_in, r).total;
}

// Forward on validated arguments.  u = x A^T has rt columns (rt = r, or
// the sum of the ranks of sibling groups, each of rank r); B has r columns;
// output rows of group i use u's columns i r .. i r + r - 1.
qn_status fwd_gemm_impl(const void* x, int64_t m, const qn_nf4_weight* w, const void* A, const void* B, int r,
                        int rt, float alpha, void* y, void* u_save, void* ws, cudaStream_t st,
                        const LoraGroups& lg) {
  const Layout L = layout(m, w->n_out, w->k_in, rt);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  if (r > 0) {
    // With SMs the GEMM leaves idle, u runs there beside the GEMM (which only
    // needs u for its last k-steps); otherwise before it on every SM.
    const int spare = side_sms<0>(m, w->n_out);
    cudaError_t e = spare > 0 ? run_lora_down_fwd(x, m, w, A, rt, lora_scale(alpha, r), u_save, L, wsb, st, false,
                                                  spare, true)
                              : run_lora_down_fwd(x, m, w, A, rt, lora_scale(alpha, r), u_save, L, wsb, st, false);
    if (e != cudaSuccess) return to_status(e);
  }
  return to_status(run_gemm<0>(x, wsb + L.scaled, B, w, m, r, y, st, r > 0, nullptr, lg));
}

qn_status fwd_gemv_impl(const void* x, int64_t m, const qn_nf4_weight* w, const void* A, const void* B, int r,
                        int rt, float alpha, void* y, void* u_save, void* ws, cudaStream_t st,
                        const LoraGroups& lg) {
  if (m > 16 || w->k_in % 256 != 0) return QN_ERR_SHAPE;
  GemvPlan g;
  if (!plan_gemv(m, w->n_out, w->k_in, rt, &g)) return QN_ERR_SHAPE;
  const Layout L = layout(m, w->n_out, w->k_in, rt);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  GemvParams p = {};
  p.codes = w->codes;
  p.qscale = w->qscale;
  p.dq_step = w->dq_step;
  p.dq_mean = w->dq_mean;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.T = static_cast<int>(m);
  p.N = w->n_out;
  p.K = w->k_in;
  p.kb = static_cast<int>(w->k_in / 64);
  p.nkr = static_cast<int>(w->k_in / 256);
  p.nrg = static_cast<int>(w->n_out / 8);
  p.rg_batch = g.rg_batch;
  p.ru_q = static_cast<int>((w->n_out / 16) / g.grid);
  p.ru_r = static_cast<int>((w->n_out / 16) % g.grid);
  std::memcpy(p.lut, gemv_lut(), sizeof(p.lut));
  // the call's first kernel: wait for the preceding work before any input
  p.wait_all = 1;
  p.lgroups = lg.count;
  p.lgcol = lg.col;
  for (int i = 0; i < 4; ++i) p.lgstart[i] = lg.start[i];
  if (r > 0) {
    // u = x A^T on the first rt / 8 CTAs of the same launch
    p.n_u = rt / 8;
    p.ur = rt;
    p.sync = reinterpret_cast<unsigned int*>(wsb + L.sync);
    p.wb = static_cast<const __nv_bfloat16*>(A);
    p.s = lora_scale(alpha, r);
    p.u_out = static_cast<__nv_bfloat16*>(u_save);
    p.us_out = reinterpret_cast<__nv_bfloat16*>(wsb + L.scaled);
    p.us_ld = static_cast<int>(round_up(rt, 64));
  }
  p.B = r > 0 ? static_cast<const __nv_bfloat16*>(B) : nullptr;
  p.us = reinterpret_cast<const __nv_bfloat16*>(wsb + L.scaled);
  p.r = r;
  p.rp = static_cast<int>(round_up(rt, 64));
  p.y = static_cast<__nv_bfloat16*>(y);
  p.lv = levels();
  CUtensorMap tm;
  if (!tmap_codes(&tm, w, 128, 16)) return to_status(cudaErrorInvalidValue);
  // a programmatic dependent launch: its CTAs set up and pull their weights
  // into L2 while the previous work drains, and wait for it before reading
  // any input
  const int grid = g.grid + p.n_u;
  const cudaError_t e = (g.nh == 1) ? run_gemv_kernel<1>(tm, p, grid, g.smem, st, true)
                                    : run_gemv_kernel<2>(tm, p, grid, g.smem, st, true);
  return to_status(e);
}

qn_status qlora_linear_fwd_gemm(const void* x, int64_t m, const qn_nf4_weight* w, const void* A,
                                const void* B, int r, float alpha, void* y, void* u_save, void* ws,
                                size_t ws_bytes, qn_stream_t stream) {
  clear_detail();
  qn_status s = validate_fwd(x, m, w, A, B, r, alpha, y, u_save, ws, ws_bytes);
  if (s != QN_OK || m == 0) return s;
  return fwd_gemm_impl(x, m, w, A, B, r, r, alpha, y, u_save, ws, reinterpret_cast<cudaStream_t>(stream),
                       LoraGroups());
}

qn_status qlora_linear_fwd_gemv(const void* x, int64_t m, const qn_nf4_weight* w, const void* A,
                                const void* B, int r, float alpha, void* y, void* u_save, void* ws,
                                size_t ws_bytes, qn_stream_t stream) {
  clear_detail();
  qn_status s = validate_fwd(x, m, w, A, B, r, alpha, y, u_save, ws, ws_bytes);
  if (s != QN_OK || m == 0) return s;
  return fwd_gemv_impl(x, m, w, A, B, r, r, alpha, y, u_save, ws, reinterpret_cast<cudaStream_t>(stream),
                       LoraGroups());
}

qn_status qlora_linear_fwd(const void* x, int64_t m, const qn_nf4_weight* w, const void* A, const void* B,
                           int r, float alpha, void* y, void* u_save, void* ws, size_t ws_bytes,
                           qn_stream_t stream) {
  if (m >= 1 && m <= 16 && w && w->k_in % 256 == 0)
    return qlora_linear_fwd_gemv(x, m, w, A, B, r, alpha, y, u_save, ws, ws_bytes, stream);
  return qlora_linear_fwd_gemm(x, m, w, A, B, r, alpha, y, u_save, ws, ws_bytes, stream);
}

// Backward on validated arguments (see fwd_gemm_impl for r, rt and the
// groups): v_i = dy_i B_i and dB_i = s dy_i^T u_i per group (dy_i: the
// group's columns of dy), dx = dy W_hat + s v A and dA = s v^T x over all rt
// rank columns.
qn_status bwd_impl(const void* dy, const void* x, int64_t m, const qn_nf4_weight* w, const void* A, const void* B,
                   int r, int rt, float alpha, const void* u, void* dx, float* dA, float* dB, void* ws,
                   cudaStream_t st, const LoraGroups& lg) {
  const Layout L = layout(m, w->n_out, w->k_in, rt);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const float sc = lora_scale(alpha, r);
  const int64_t N = w->n_out, K = w->k_in;
  const int G = lg.count;
  const int rpt = static_cast<int>(round_up(rt, 64));
  cudaError_t e = cudaSuccess;
  if (r == 0) {
    if (dx) e = run_gemm<1>(dy, wsb + L.scaled, A, w, m, r, dx, st, false);
    return to_status(e);
  }
  const __nv_bfloat16* dyb = static_cast<const __nv_bfloat16*>(dy);
  const __nv_bfloat16* Bb = static_cast<const __nv_bfloat16*>(B);
  __nv_bfloat16* vplain = reinterpret_cast<__nv_bfloat16*>(wsb + L.vplain);
  __nv_bfloat16* vscaled = reinterpret_cast<__nv_bfloat16*>(wsb + L.scaled);
  // v = dy B per group (and u = x A^T when the forward's u is not given).
  // With u given and SMs the dx GEMM leaves idle, v runs there beside the
  // GEMM, which needs it only for its last k-blocks, and dA / dB follow the
  // GEMM; otherwise v (and u), then dA / dB, then the GEMM.
  SmallProblem pr[kSmallMaxProblems + 1];
  int count = 0;
  for (int i = 0; i < G; ++i) {
    const int64_t n0 = lg.start[i], ni = (i + 1 < G ? lg.start[i + 1] : N) - n0;
    SmallProblem& P = pr[count++];
    P = small_problem(0, dyb + n0, Bb + n0 * r, 1, m, ni, r, sc);
    P.ldx = N;
    P.plain = vplain + i * r;
    P.ldp = rt;
    P.scaled = vscaled + i * r;
    P.rp = rpt;
    P.pad = i + 1 == G ? rpt - rt : 0;
  }
  const void* u_use = u;
  if (!u) {
    SmallProblem& P = pr[count++];
    P = small_problem(0, x, A, 0, m, K, rt, sc);
    P.plain = reinterpret_cast<__nv_bfloat16*>(wsb + L.uplain);
    u_use = wsb + L.uplain;
  }
  // dB_i = s dy_i^T u_i ([n_i, r]) per group.
  const __nv_bfloat16* ub = static_cast<const __nv_bfloat16*>(u_use);
  SmallProblem db[kMaxSiblingGroups];
  for (int i = 0; i < G; ++i) {
    const int64_t n0 = lg.start[i], ni = (i + 1 < G ? lg.start[i + 1] : N) - n0;
    db[i] = small_problem(1, dyb + n0, ub + i * r, 0, ni, m, r, sc);
    db[i].ldx = N;
    db[i].ldw = rt;
    db[i].out = dB + n0 * r;
    db[i].transpose = 0;
  }
  // With u given and SMs the dx GEMM leaves idle, v runs there beside the
  // GEMM (which needs it only for its last k-blocks) and dA / dB follow the
  // GEMM; otherwise v (and u), then dA / dB, then the GEMM.  (dA and dB
  // beside the GEMM would take longer than it: a rank-r CTA streams far
  // slower than an SM's share of HBM, and they read twice the bytes of v.)
  const int spare = (dx && u) ? side_sms<1>(m, K) : 0;
  e = run_small_by_rank(pr, count, st, false, spare);
  if (e != cudaSuccess) return to_status(e);
  if (dx && spare > 0) {
    e = run_gemm<1>(dy, vscaled, A, w, m, rt, dx, st, true);
    if (e != cudaSuccess) return to_status(e);
  }
  // dA^T = s x^T v  ([K, rt], stored transposed as dA [rt, K]) and dB, on
  // every SM.
  SmallProblem up[kSmallMaxProblems + 1];
  int nup = 0;
  up[nup] = small_problem(1, x, vplain, 0, K, m, rt, sc);
  up[nup].out = dA;
  up[nup].transpose = 1;
  ++nup;
  for (int i = 0; i < G; ++i) up[nup++] = db[i];
  e = run_small_by_rank(up, nup, st, true, 0);
  if (e != cudaSuccess) return to_status(e);
  if (dx && spare == 0) {
    e = run_gemm<1>(dy, vscaled, A, w, m, rt, dx, st, true);
    if (e != cudaSuccess) return to_status(e);
  }
  return QN_OK;
}

qn_status qlora_linear_bwd(const void* dy, const void* x, int64_t m, const qn_nf4_weight* w, const void* A,
                           const void* B, int r, float alpha, const void* u, void* dx, float* dA, float* dB,
                           void* ws, size_t ws_bytes, qn_stream_t stream) {
  clear_detail();
  qn_status s = check_layer(w, r);
  if (s != QN_OK) return s;
  if (m < 0) return QN_ERR_SHAPE;
  if (m == 0) return QN_OK;
  if (!dy) return QN_ERR_ARG;
  if (r > 0 && (!x || !A || !B || !dA || !dB || !std::isfinite(alpha))) return QN_ERR_ARG;
  if (!aligned16(dy) || (dx && !aligned16(dx)) || (x && !aligned16(x)) ||
      (r > 0 && (!aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB))) ||
      (u && !aligned16(u)))
    return QN_ERR_ALIGN;
  const Layout L = layout(m, w->n_out, w->k_in, r);
  if (!ws || ws_bytes < L.total) return QN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  return bwd_impl(dy, x, m, w, A, B, r, r, alpha, u, dx, dA, dB, ws, reinterpret_cast<cudaStream_t>(stream),
                  LoraGroups());
}

// ------------------------------------------------------------------ sibling linears

// Checks the sibling groups against the stacked weight; fills the LoRA
// groups (row starts, column stride r).
qn_status sibling_groups(const qn_nf4_weight* w, int groups, const int64_t* rows, int r, LoraGroups* lg) {
  if (!w || !rows) return QN_ERR_ARG;
  if (groups < 1 || groups > kMaxSiblingGroups) return QN_ERR_SHAPE;
  if (r < 8 || r % 8 != 0 || static_cast<int64_t>(groups) * r > kMaxRank) return QN_ERR_SHAPE;
  int64_t total = 0;
  lg->count = groups;
  lg->col = r;
  for (int i = 0; i < groups; ++i) {
    if (rows[i] <= 0 || rows[i] % 256 != 0) return QN_ERR_SHAPE;
    lg->start[i] = total;
    total += rows[i];
  }
  if (total != w->n_out) return QN_ERR_SHAPE;
  return QN_OK;
}

size_t qlora_siblings_workspace_bytes(int64_t m, int64_t n_total, int64_t k_in, int groups, int r) {
  if (m < 0 || n_total <= 0 || k_in <= 0 || groups < 1 || r < 0) return 0;
  return layout(m, n_total, k_in, groups * r).total;
}

qn_status qlora_siblings_fwd(const void* x, int64_t m, const qn_nf4_weight* w, int groups, const int64_t* rows,
                             const void* A, const void* B, int r, float alpha, void* y, void* u_save, void* ws,
                             size_t ws_bytes, qn_stream_t stream) {
  clear_detail();
  LoraGroups lg;
  qn_status s = sibling_groups(w, groups, rows, r, &lg);
  if (s != QN_OK) return s;
  const int rt = groups * r;
  s = validate_fwd(x, m, w, A, B, rt, alpha, y, u_save, ws, ws_bytes);
  if (s != QN_OK || m == 0) return s;
  lg.width = round_up(rt, 64);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (m <= 16 && w->k_in % 256 == 0) return fwd_gemv_impl(x, m, w, A, B, r, rt, alpha, y, u_save, ws, st, lg);
  return fwd_gemm_impl(x, m, w, A, B, r, rt, alpha, y, u_save, ws, st, lg);
}

qn_status qlora_siblings_bwd(const void* dy, const void* x, int64_t m, const qn_nf4_weight* w, int groups,
                             const int64_t* rows, const void* A, const void* B, int r, float alpha, const void* u,
                             void* dx, float* dA, float* dB, void* ws, size_t ws_bytes, qn_stream_t stream) {
  clear_detail();
  LoraGroups lg;
  qn_status s = sibling_groups(w, groups, rows, r, &lg);
  if (s != QN_OK) return s;
  const int rt = groups * r;
  s = check_layer(w, rt);
  if (s != QN_OK) return s;
  if (m < 0) return QN_ERR_SHAPE;
  if (m == 0) return QN_OK;
  if (!dy || !x || !A || !B || !dA || !dB || !std::isfinite(alpha)) return QN_ERR_ARG;
  if (!aligned16(dy) || (dx && !aligned16(dx)) || !aligned16(x) || !aligned16(A) || !aligned16(B) ||
      !aligned16(dA) || !aligned16(dB) || (u && !aligned16(u)))
    return QN_ERR_ALIGN;
  const Layout L = layout(m, w->n_out, w->k_in, rt);
  if (!ws || ws_bytes < L.total) return QN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  lg.width = round_up(rt, 64);
  return bwd_impl(dy, x, m, w, A, B, r, rt, alpha, u, dx, dA, dB, ws, reinterpret_cast<cudaStream_t>(stream), lg);
}

qn_status qlora_merge(const qn_nf4_weight* w, const void* A, const void* B, int r, float alpha, void* w_out,
                      qn_stream_t stream) {
  clear_detail();
  qn_status s = check_layer(w, r);
  if (s != QN_OK) return s;
  if (!w_out || (r > 0 && (!A || !B || !std::isfinite(alpha)))) return QN_ERR_ARG;
  if (!aligned16(w_out) || (r > 0 && (!aligned16(A) || !aligned16(B)))) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  static std::once_flag once;
  static bool ok = false;
  std::call_once(once, [] { ok = set_smem(qlora_merge_kernel, merge_smem_bytes(kMaxRank)); });
  if (!ok) return to_status(cudaErrorInvalidValue);
  MergeParams p = {};
  p.codes = w->codes;
  p.qscale = w->qscale;
  p.dq_step = w->dq_step;
  p.dq_mean = w->dq_mean;
  p.A = static_cast<const __nv_bfloat16*>(A);
  p.B = static_cast<const __nv_bfloat16*>(B);
  p.out = static_cast<__nv_bfloat16*>(w_out);
  p.N = w->n_out;
  p.K = w->k_in;
  p.r = r;
  p.s = lora_scale(alpha, r);
  p.lv = levels();
  // persistent CTAs: as many as fit on the device at once, or one per tile
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qlora_merge_kernel, kMergeThreads,
                                                    merge_smem_bytes(r)) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t tiles = ceil_div(w->k_in, kMergeCols) * (w->n_out / kMergeRows);
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, static_cast<int64_t>(per_sm) * sm_count()));
  return to_status(launch(qlora_merge_kernel, dim3(grid), dim3(kMergeThreads), merge_smem_bytes(r),
                          reinterpret_cast<cudaStream_t>(stream), false, p));
}

size_t qlora_adamw8_blocks(int64_t n) { return n > 0 ? static_cast<size_t>((n + kAdamBlock - 1) / kAdamBlock) : 0; }

qn_status qlora_adamw8_step(float* param, const float* grad, int64_t n, uint8_t* m_codes, float* m_scale,
                            uint8_t* v_codes, float* v_scale, void* param_bf16, float lr, float beta1, float beta2,
                            float eps, float weight_decay, int64_t step, qn_stream_t stream) {
  clear_detail();
  if (n < 0) return QN_ERR_SHAPE;
  const bool hp_ok = std::isfinite(lr) && lr >= 0.f && std::isfinite(beta1) && beta1 >= 0.f && beta1 < 1.f &&
                     std::isfinite(beta2) && beta2 >= 0.f && beta2 < 1.f && std::isfinite(eps) && eps > 0.f &&
                     std::isfinite(weight_decay) && weight_decay >= 0.f && step >= 1;
  if (!hp_ok) return QN_ERR_ARG;
  if (n == 0) return QN_OK;
  if (!param || !grad || !m_codes || !m_scale || !v_codes || !v_scale) return QN_ERR_ARG;
  if (!aligned16(param) || !aligned16(grad) || !aligned16(m_codes) || !aligned16(m_scale) ||
      !aligned16(v_codes) || !aligned16(v_scale) || (param_bf16 && !aligned16(param_bf16)))
    return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  AdamW8Params a = {};
  a.p = param;
  a.g = grad;
  a.mc = m_codes;
  a.ms = m_scale;
  a.vc = v_codes;
  a.vs = v_scale;
  a.pb = static_cast<__nv_bfloat16*>(param_bf16);
  a.n = n;
  // fp64 on the host from the fp32 hyperparameters, rounded once
  const double b1 = beta1, b2 = beta2;
  a.b1 = beta1;
  a.b2 = beta2;
  a.omb1 = static_cast<float>(1.0 - b1);
  a.omb2 = static_cast<float>(1.0 - b2);
  const double bc1 = 1.0 - std::pow(b1, static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(b2, static_cast<double>(step));
  if (!(bc1 > 0.0) || !(bc2 > 0.0)) return QN_ERR_ARG;     // beta^t rounds to 1: no step is possible
  a.step_size = static_cast<float>(static_cast<double>(lr) / bc1);
  a.rsqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
  a.decay = static_cast<float>(1.0 - static_cast<double>(lr) * static_cast<double>(weight_decay));
  a.eps = eps;
  const int64_t nblk = (n + kAdamBlock - 1) / kAdamBlock;
  // one wave of resident CTAs, each looping over blocks
  static int per_sm = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adamw8_kernel, kAdamThreads, 0) != cudaSuccess)
      per_sm = 4;
  });
  const int64_t grid = std::min<int64_t>(ceil_div(nblk, kAdamThreads / 32),
                                         static_cast<int64_t>(std::max(per_sm, 1)) * sm_count());
  return to_status(launch(adamw8_kernel, dim3(static_cast<unsigned>(grid)), dim3(kAdamThreads), 0,
                          reinterpret_cast<cudaStream_t>(stream), false, a));
}

size_t qlora_dropout_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int r) {
  if (m < 0 || n_out <= 0 || k_in <= 0 || r < 0) return 0;
  return layout(m, n_out, k_in, r, true).total;
}

qn_status lora_dropout(const void* x, int64_t m, int64_t k, float p, uint64_t seed, uint64_t offset, void* x_drop,
                       uint32_t* keep, qn_stream_t stream) {
  clear_detail();
  if (m < 0 || k <= 0 || k % 32 != 0) return QN_ERR_SHAPE;
  if (!dropout_rate_ok(p)) return QN_ERR_ARG;
  if (m == 0) return QN_OK;
  if (!x || !x_drop || !keep) return QN_ERR_ARG;
  if (!aligned16(x) || !aligned16(x_drop) || !aligned16(keep)) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  return to_status(run_dropout(x, m, k, p, seed, offset, x_drop, keep, reinterpret_cast<cudaStream_t>(stream)));
}

qn_status qlora_linear_fwd_dropout(const void* x, int64_t m, const qn_nf4_weight* w, const void* A, const void* B,
                                   int r, float alpha, float p, uint64_t seed, uint64_t offset, void* y,
                                   void* u_save, void* x_drop, uint32_t* keep, void* ws, size_t ws_bytes,
                                   qn_stream_t stream) {
  clear_detail();
  if (r <= 0 || !dropout_rate_ok(p)) return QN_ERR_ARG;
  if (m > 0 && (!x_drop || !keep)) return QN_ERR_ARG;
  if (m > 0 && (!aligned16(x_drop) || !aligned16(keep))) return QN_ERR_ALIGN;
  qn_status s = validate_fwd(x, m, w, A, B, r, alpha, y, u_save, ws, ws_bytes, true);
  if (s != QN_OK || m == 0) return s;
  const Layout L = layout(m, w->n_out, w->k_in, r, true);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const float sd = dropout_scale(lora_scale(alpha, r), p);
  // x_m and the mask; then u = x_m A^T (beside the GEMM on the SMs it leaves
  // idle, when there are some), waiting for x_m; then the GEMM, which reads
  // x itself and waits for u only before its LoRA k-block.
  cudaError_t e = run_dropout(x, m, w->k_in, p, seed, offset, x_drop, keep, st);
  if (e != cudaSuccess) return to_status(e);
  const int spare = side_sms<0>(m, w->n_out);
  // u starts after the mask kernel has left every SM (no early launch), so
  // that its CTAs take SMs the GEMM's clusters can spare, as in the plain path
  e = spare > 0 ? run_lora_down_fwd(x_drop, m, w, A, r, sd, u_save, L, wsb, st, false, spare, true)
                : run_lora_down_fwd(x_drop, m, w, A, r, sd, u_save, L, wsb, st, true);
  if (e != cudaSuccess) return to_status(e);
  return to_status(run_gemm<0>(x, wsb + L.scaled, B, w, m, r, y, st, true));
}

qn_status qlora_linear_bwd_dropout(const void* dy, const void* x_drop, const uint32_t* keep, int64_t m,
                                   const qn_nf4_weight* w, const void* A, const void* B, int r, float alpha,
                                   float p, const void* u, void* dx, float* dA, float* dB, void* ws,
                                   size_t ws_bytes, qn_stream_t stream) {
  clear_detail();
  qn_status s = check_layer(w, r);
  if (s != QN_OK) return s;
  if (r <= 0 || !dropout_rate_ok(p) || !std::isfinite(alpha)) return QN_ERR_ARG;
  if (m < 0) return QN_ERR_SHAPE;
  if (m == 0) return QN_OK;
  if (!dy || !x_drop || !A || !B || !dA || !dB || (dx && !keep)) return QN_ERR_ARG;
  if (!aligned16(dy) || !aligned16(x_drop) || !aligned16(A) || !aligned16(B) || !aligned16(dA) ||
      !aligned16(dB) || (dx && (!aligned16(dx) || !aligned16(keep))) || (u && !aligned16(u)))
    return QN_ERR_ALIGN;
  const Layout L = layout(m, w->n_out, w->k_in, r, true);
  if (!ws || ws_bytes < L.total) return QN_ERR_WORKSPACE;
  if (!aligned16(ws)) return QN_ERR_ALIGN;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const float sd = dropout_scale(lora_scale(alpha, r), p);
  const int64_t N = w->n_out, K = w->k_in;
  float* dxf = reinterpret_cast<float*>(wsb + L.dxf);
  // v = dy B (and u = x_m A^T when not given), on the SMs the base GEMM
  // leaves idle when it leaves some and u is given, else before it; the base
  // GEMM dy W_hat (fp32), which waits for v before exiting; dA, dB; then
  // dx = bf16(base + s_d keep (v A)).  Each kernel after the first waits for
  // the one before it, so the last one's completion implies all.
  cudaError_t e = cudaSuccess;
  SmallProblem pr[2];
  pr[0] = small_problem(0, dy, B, 1, m, N, r, sd);
  pr[0].plain = reinterpret_cast<__nv_bfloat16*>(wsb + L.vplain);
  pr[0].scaled = reinterpret_cast<__nv_bfloat16*>(wsb + L.scaled);
  int count = 1;
  const void* u_use = u;
  if (!u) {
    pr[1] = small_problem(0, x_drop, A, 0, m, K, r, sd);
    pr[1].plain = reinterpret_cast<__nv_bfloat16*>(wsb + L.uplain);
    u_use = wsb + L.uplain;
    count = 2;
  }
  const int spare = (dx && u) ? side_sms<1, true>(m, K) : 0;
  e = spare > 0 ? run_small(pr, count, st, false, spare, true) : run_small(pr, count, st, false);
  if (e != cudaSuccess) return to_status(e);
  if (dx) {
    e = run_gemm<1, true>(dy, wsb + L.scaled, A, w, m, 0, nullptr, st, true, dxf);
    if (e != cudaSuccess) return to_status(e);
  }
  SmallProblem up[2];
  up[0] = small_problem(1, x_drop, wsb + L.vplain, 0, K, m, r, sd);
  up[0].out = dA;
  up[0].transpose = 1;
  up[1] = small_problem(1, dy, u_use, 0, N, m, r, sd);
  up[1].out = dB;
  up[1].transpose = 0;
  e = run_small(up, 2, st, true);
  if (e != cudaSuccess) return to_status(e);
  if (dx) e = run_dx_dropout(dxf, keep, wsb + L.vplain, A, dx, m, K, r, sd, st);
  return to_status(e);
}

}  // extern "C"

// ====================================================================== no-allocation quantize
//
// nf4_quantize needs one fp32 scratch value per block of 64 weights (the
// exact absmax, read back by the second-level pass).  Some callers cannot
// hand over that workspace: code that runs where allocating device memory
// is not allowed once the program is up (a runtime whose memory was planned
// and reserved at start-up, or a plug-in that only sees buffers its host
// framework gives it), or callers that have no allocator of their own.  For
// them the scratch lives in this file-scope array instead, kNoallocMaxBlocks
// values (4 MiB), which every GPU that loads this library holds until the
// process exits.  The kernels are the same as nf4_quantize's; only where the
// scratch comes from differs.

namespace {

constexpr int64_t kNoallocMaxBlocks = int64_t{1} << 20;   // 64 Mi weights at most

static __device__ __align__(256) float g_noalloc_absmax[kNoallocMaxBlocks];

// Host code cannot use g_noalloc_absmax as a device address (the name is a
// host-side stand-in); its device address is looked up once per device,
// with that device current, and cached.
std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[64] = {};

qn_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return to_status(e);
  if (dev < 0 || dev >= 64) return QN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_absmax);
    if (e != cudaSuccess || p == nullptr) return to_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return QN_OK;
}

}  // namespace

extern "C" qn_status nf4_quantize_noalloc(const void* w_bf16, const qn_nf4_weight* out, qn_stream_t stream) {
  clear_detail();
  qn_status s = check_weight(out);
  if (s != QN_OK) return s;
  if (!w_bf16) return QN_ERR_ARG;
  if (!aligned16(w_bf16)) return QN_ERR_ALIGN;
  const int64_t nblk = out->n_out * (out->k_in / 64);
  if (nblk > kNoallocMaxBlocks) return QN_ERR_SHAPE;
  if (!device_is_sm100()) return QN_ERR_UNSUPPORTED;
  float* absmax = nullptr;
  s = noalloc_scratch(&absmax);
  if (s != QN_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t ngroups = ceil_div(nblk, 256);
  cudaError_t e = run_encode(w_bf16, out, absmax, nblk, st);
  if (e != cudaSuccess) return to_status(e);
  e = launch(nf4_dq_kernel, dim3(static_cast<unsigned>(ceil_div(ngroups, 8))), dim3(256), 0, st, false,
             static_cast<const float*>(absmax), nblk, out->qscale, out->dq_step, out->dq_mean, ngroups);
  return to_status(e);
}
