/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so: the QLoRA frozen linear layer on
 * NVIDIA B200 (sm_100a).
 *
 * The layer keeps a frozen weight W [n_out, k_in] as 4-bit NormalFloat codes
 * with one absmax scale per block of 64 weights; the block scales are stored
 * again as int8 in groups of 256 (double quantization).  The forward pass
 * dequantizes W to bf16 just before the matmul and adds a LoRA path:
 *     y = x W^T + s (x A^T) B^T,   s = alpha / r,
 * with A [r, k_in] and B [n_out, r] in bf16.  The backward pass sends the
 * gradient through the dequantized W to dx and gives gradients to A and B
 * only; W gets none.
 *
 * Source passages (page title, section):
 *   Ultralytics glossary "QLoRA", "Come funziona QLoRA": NF4 codes pointing at
 *     16 normal-quantile levels, an absmax scale per block of 64, scales
 *     re-quantized to 8 bits in blocks of 256, dequantization to bfloat16 just
 *     before the matmul plus the LoRA output, backpropagation through the
 *     dequantized weights updating only the two LoRA matrices; the NF4 snippet
 *     (level construction, absmax, nearest level, restore).
 *   skyvanguard "LoRA y QLoRA en Profundidad", "Cómo Funciona LoRA" (shapes of
 *     A and B, delta_W = B @ A) and "Alpha (lora_alpha)" (scale alpha / r);
 *     the QLoRA config (compute dtype bfloat16, double quantization on).
 *   "Módulo 4: QLoRA", 4.2 (4 bits = half a byte per weight), 4.3 b) (scale
 *     constants quantized to 8 bits), 4.4 (only A and B train).
 *
 * Storage layout (decisions where the pages are silent):
 *   codes   uint8 [n_out, k_in/2] row-major; byte j of a row holds element 2j
 *           in its low nibble and element 2j+1 in its high nibble.
 *   qscale  int8  [nblk], nblk = n_out*k_in/64, one per 64 consecutive weights
 *           of a row (flattened row-major order).
 *   dq_step, dq_mean  float32 [ngroups], ngroups = ceil(nblk/256): group g
 *           covers qscale[256g .. 256g+255]; the block scale is restored as
 *           s_hat = fl32(fl32(q * dq_step[g]) + dq_mean[g]).
 *   W_hat = bf16_rne(fl32(level[code] * s_hat)), level = the 16 NF4 values.
 *
 * Conventions for every call:
 *   - Every pointer is a DEVICE pointer unless stated otherwise, owned by the
 *     caller, 16-byte aligned; the library allocates no device memory and
 *     keeps no state between calls except the device error word below.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously.  Argument errors are reported before
 *     anything is enqueued.  A failed launch returns QN_ERR_CUDA.
 *   - bf16 tensors are row-major with no padding: x [M, k_in], y [M, n_out],
 *     dy [M, n_out], dx [M, k_in], A [r, k_in], B [n_out, r].
 *   - Shapes: k_in % 64 == 0 and n_out % 64 == 0 (QN_ERR_SHAPE otherwise);
 *     the LoRA rank r is 0 (no LoRA path) or a multiple of 8 in [8, 128];
 *     M >= 0 (M == 0 enqueues nothing).
 *   - Waits inside kernels are bounded; a wait that gives up sets a bit in the
 *     device error word (read with qn_device_error) and the call's outputs
 *     are then undefined.
 *   - Concurrent calls that share a workspace race; give each stream its own.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI version, bumped on any incompatible change of this header. */
#define QN_ABI_VERSION 1

typedef struct CUstream_st* qn_stream_t;   /* same type as cudaStream_t */

typedef enum {
  QN_OK = 0,
  QN_ERR_ARG = 1,            /* NULL pointer or invalid scalar argument     */
  QN_ERR_SHAPE = 2,          /* unsupported sizes (see conventions above)   */
  QN_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned            */
  QN_ERR_WORKSPACE = 4,      /* workspace NULL or smaller than required     */
  QN_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed        */
  QN_ERR_DEVICE_TIMEOUT = 6, /* a bounded device wait gave up               */
  QN_ERR_UNSUPPORTED = 7     /* the current device is not sm_100            */
} qn_status;

/* A quantized weight.  All array pointers are device pointers (see layout). */
typedef struct {
  int64_t n_out;        /* rows of W (d_out)                      */
  int64_t k_in;         /* columns of W (d_in), multiple of 64    */
  uint8_t* codes;       /* [n_out, k_in/2]                        */
  int8_t* qscale;       /* [n_out*k_in/64]                        */
  float* dq_step;       /* [ceil(n_out*k_in/64/256)]              */
  float* dq_mean;       /* [ceil(n_out*k_in/64/256)]              */
} qn_nf4_weight;

/* Returns QN_ABI_VERSION. */
int qn_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* qn_status_string(qn_status status);

/* Name of the last CUDA error behind a QN_ERR_CUDA returned on this host
 * thread ("no error" if none); a static string, never NULL. */
const char* qn_last_error_string(void);

/* Writes the 16 NF4 levels (fp32, ascending, level[7] == 0) to HOST memory
 * `out`.  The table is the normal-quantile construction of the QLoRA
 * glossary's NF4 snippet, evaluated in fp64 and rounded once to fp32. */
void nf4_levels(float out[16]);

/* Reads and clears the device error word on the current device (blocking:
 * synchronizes the device first).  *flags_out (HOST) receives the OR of the
 * bits set since the last read; 0 means no bounded wait gave up.  Bits: 1 a
 * wait of the tensor-core GEMM, 2 of the decode GEMV, 4 of a rank-r kernel,
 * QN_WAIT_SELFTEST of qn_selftest_bounded_wait. */
qn_status qn_device_error(int* flags_out);

/* Failure-detection self-test: enqueues one warp whose thread 0 waits on a
 * barrier phase that nothing completes, with the same bounded wait as the
 * library's pipelines.  The wait gives up after the limit (2 s of device
 * time), sets QN_WAIT_SELFTEST in the device error word, and the kernel
 * returns: the context stays usable.  For tests that check that a stuck wait
 * is reported rather than left hanging. */
#define QN_WAIT_SELFTEST 8
qn_status qn_selftest_bounded_wait(qn_stream_t stream);

/* ---------------------------------------------------------------- storage */

/* Bytes of workspace nf4_quantize needs: one fp32 absmax per block of 64. */
size_t nf4_quantize_workspace_bytes(int64_t n_out, int64_t k_in);

/* Quantizes bf16 W [n_out, k_in] into `out` (whose n_out/k_in must match and
 * whose arrays the caller allocated with the sizes above).
 * [QLoRA glossary, "Come funziona QLoRA" and NF4 snippet: per block of 64,
 * absmax; x = w / absmax in fp32; code = the first level index minimising
 * |x - level| in fp32.  Then per group of 256 block scales: mean = the fp64
 * sum / count rounded to fp32, step = max|s - mean| / 127, q = round-half-even
 * ((s - mean) / step) in [-127, 127] ("Doppia quantizzazione").]
 * An all-zero block gets scale 0 and zero-level codes.  Codes, qscale,
 * dq_step and dq_mean are bit-identical to the CPU definition.
 * ws: device workspace of at least nf4_quantize_workspace_bytes bytes. */
qn_status nf4_quantize(const void* w_bf16, const qn_nf4_weight* out,
                       void* ws, size_t ws_bytes, qn_stream_t stream);

/* nf4_quantize for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is an interface choice of the library.
 * Some callers cannot give a workspace: code running where device
 * allocation is no longer allowed once the program is up (memory planned
 * and reserved at start-up, or a plug-in that only sees the buffers its
 * host framework passes in), or code with no allocator of its own.  This
 * call takes no workspace and allocates nothing; its fp32 scratch (one value
 * per block of 64 weights) is a fixed array inside the library of
 * 2^20 values (4 MiB, at most 64 Mi weights, i.e. n_out * k_in / 64 <=
 * 1048576), held on every GPU that loads the library until the process
 * exits.  Larger weights return QN_ERR_SHAPE before any work is enqueued.
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture on that device.  All calls share the one array and leave their
 * values in it (nothing in it needs to start at zero: a call writes every
 * entry it reads): calls that overlap on the GPU (other streams, other host
 * threads) race, so serialize them.  Results are bit-identical to
 * nf4_quantize's. */
qn_status nf4_quantize_noalloc(const void* w_bf16, const qn_nf4_weight* out, qn_stream_t stream);

/* Writes W_hat (bf16 [n_out, k_in]) = bf16_rne(level[code] * s_hat), bit-exact.
 * [QLoRA glossary, "Come funziona QLoRA": dequantization to bfloat16] */
qn_status nf4_dequantize(const qn_nf4_weight* w, void* w_hat_bf16, qn_stream_t stream);

/* ---------------------------------------------------------------- layer */

/* Workspace for qlora_linear_fwd / qlora_linear_bwd (and the two forward
 * paths below) at these sizes; the same buffer serves both directions.  Its
 * last 256 bytes hold the decode path's counters: zero them once when the
 * workspace is made (e.g. cudaMemset); every call leaves them zero. */
size_t qlora_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int r);

/* Forward: y = x W_hat^T + s (x A^T) B^T with s = fl32(alpha / r).
 * [QLoRA glossary, "Come funziona QLoRA"; skyvanguard lesson, "Cómo Funciona
 * LoRA" and "Alpha (lora_alpha)"]
 * x bf16 [m, k_in]; A bf16 [r, k_in]; B bf16 [n_out, r]; y bf16 [m, n_out].
 * r == 0 (A, B ignored, may be NULL) computes the base path only.
 * u_save: NULL, or bf16 [m, r] receiving u = x A^T for the backward.
 * Products accumulate in fp32; y is rounded once to bf16.
 * m <= 16 with k_in % 256 == 0 runs the decode path (one launch: a GEMV
 * that streams the codes once, with u = x A^T on r / 8 of its CTAs), any
 * other m the tensor-core GEMM with
 * the dequantization fused into its operand staging (the CTAs of a cluster
 * decode each weight tile once between them). */
qn_status qlora_linear_fwd(const void* x, int64_t m, const qn_nf4_weight* w,
                           const void* A, const void* B, int r, float alpha,
                           void* y, void* u_save,
                           void* ws, size_t ws_bytes, qn_stream_t stream);

/* The two forward paths, callable directly (same arguments and result as
 * qlora_linear_fwd).  The GEMV path accepts 1 <= m <= 16 and k_in % 256 == 0
 * (QN_ERR_SHAPE otherwise). */
qn_status qlora_linear_fwd_gemm(const void* x, int64_t m, const qn_nf4_weight* w,
                                const void* A, const void* B, int r, float alpha,
                                void* y, void* u_save,
                                void* ws, size_t ws_bytes, qn_stream_t stream);
qn_status qlora_linear_fwd_gemv(const void* x, int64_t m, const qn_nf4_weight* w,
                                const void* A, const void* B, int r, float alpha,
                                void* y, void* u_save,
                                void* ws, size_t ws_bytes, qn_stream_t stream);

/* Backward of the forward above for an upstream gradient dy bf16 [m, n_out]:
 *   dx = dy W_hat + s (dy B) A          (bf16 [m, k_in]; skipped if dx NULL)
 *   dA = s (dy B)^T x                   (fp32 [r, k_in])
 *   dB = s dy^T (x A^T)                 (fp32 [n_out, r])
 * [QLoRA glossary, "Come funziona QLoRA": gradients through the dequantized
 * weights, only the two LoRA matrices updated; "Módulo 4: QLoRA", 4.4]
 * u: NULL (recomputed from x and A) or the u_save of the forward.
 * With r == 0 only dx is computed (dA, dB, A, B, u ignored). */
qn_status qlora_linear_bwd(const void* dy, const void* x, int64_t m,
                           const qn_nf4_weight* w, const void* A, const void* B,
                           int r, float alpha, const void* u,
                           void* dx, float* dA, float* dB,
                           void* ws, size_t ws_bytes, qn_stream_t stream);

/* ---------------------------------------------------------------- sibling linears */

/* Sibling linears: `groups` layers that read the same x (q, k and v of
 * attention; gate and up of the MLP), each a frozen NF4 weight W_i [n_i, k_in]
 * with its own LoRA adapter A_i [r, k_in], B_i [n_i, r] of the same rank r
 * and alpha, run as one call:
 *   y_i = x W_hat_i^T + s (x A_i^T) B_i^T,   s = fl32(alpha / r),
 * with y = [y_1 | y_2 | ...] (columns), every sibling's LoRA path at its own
 * rank r.
 * [skyvanguard lesson, "Módulos Objetivo": LoRA on q_proj, k_proj, v_proj,
 *  o_proj, or on every linear layer including gate_proj, up_proj and
 *  down_proj; QLoRA glossary, "Come funziona QLoRA": each is the frozen NF4
 *  weight plus its LoRA path.]
 * w: the siblings' NF4 weights stacked by rows ([sum n_i, k_in]; codes and
 * block scales concatenated, which is the storage of the stacked weight when
 * each n_i * k_in / 64 is a multiple of 256); rows: HOST array of the n_i,
 * 1 <= groups <= 4, each n_i a multiple of 256, their sum w->n_out;
 * A bf16 [groups * r, k_in] (the A_i stacked); B bf16 [sum n_i, r] (the B_i
 * stacked); y bf16 [m, sum n_i]; u_save NULL or bf16 [m, groups * r].
 * r a multiple of 8 with groups * r <= 128 (QN_ERR_SHAPE otherwise).  The
 * workspace is qlora_siblings_workspace_bytes, its last 256 bytes zeroed
 * once when made.  Results equal those of one qlora_linear_fwd per sibling
 * up to the order of fp32 accumulation. */
size_t qlora_siblings_workspace_bytes(int64_t m, int64_t n_total, int64_t k_in, int groups, int r);
qn_status qlora_siblings_fwd(const void* x, int64_t m, const qn_nf4_weight* w, int groups, const int64_t* rows,
                             const void* A, const void* B, int r, float alpha, void* y, void* u_save,
                             void* ws, size_t ws_bytes, qn_stream_t stream);

/* Backward of qlora_siblings_fwd for dy = [dy_1 | dy_2 | ...] bf16
 * [m, sum n_i]: dx = sum_i (dy_i W_hat_i + s (dy_i B_i) A_i) (bf16 [m, k_in];
 * skipped if dx NULL), dA = the dA_i stacked (fp32 [groups * r, k_in]),
 * dB = the dB_i stacked (fp32 [sum n_i, r]); each dA_i, dB_i as
 * qlora_linear_bwd gives them.  u: NULL or the forward's u_save.  Other
 * arguments as for qlora_siblings_fwd. */
qn_status qlora_siblings_bwd(const void* dy, const void* x, int64_t m, const qn_nf4_weight* w, int groups,
                             const int64_t* rows, const void* A, const void* B, int r, float alpha,
                             const void* u, void* dx, float* dA, float* dB,
                             void* ws, size_t ws_bytes, qn_stream_t stream);

/* ---------------------------------------------------------------- merge */

/* Folds the LoRA adapter into the dequantized weight:
 *   w_out = bf16( W_hat + fl32(s * (B A)) ),  s = fl32(alpha / r),
 * with W_hat = bf16(level[code] * s_hat) (bit-identical to nf4_dequantize),
 * B A accumulated in fp32 and one bf16 rounding of the fp32 sum.
 * [skyvanguard lesson, "Cómo Funciona LoRA": for inference the LoRA matrices
 * are merged, W_final = W + (alpha / r) B @ A; QLoRA glossary, "Compromessi":
 * merging into the 4-bit base first dequantizes it to 16 bits; "QLoRA e
 * metodi correlati": the merged 16-bit weights are often quantized again,
 * which is nf4_quantize of w_out.]
 * w: the NF4 weight [n_out, k_in]; A bf16 [r, k_in]; B bf16 [n_out, r];
 * w_out bf16 [n_out, k_in] (DEVICE, caller-owned).  r == 0 (A, B ignored,
 * may be NULL) writes W_hat.  Shape rules as for the layer calls. */
qn_status qlora_merge(const qn_nf4_weight* w, const void* A, const void* B, int r, float alpha,
                      void* w_out, qn_stream_t stream);

/* ---------------------------------------------------------------- dropout */

/* LoRA dropout: the LoRA path reads dropout(x) = x * keep / (1 - p) instead
 * of x, the base path reads x.
 * [skyvanguard lesson, "Dropout (lora_dropout)": the LoRA layers' dropout
 *  zeroes randomly chosen elements during training as regularisation; 0.05
 *  in the lesson's config.]
 * The draw is Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random
 * Numbers: As Easy as 1, 2, 3", SC 2011): element e = i * k + j of x [m, k]
 * takes word e % 4 of the block with counter (lo32(e/4), hi32(e/4),
 * lo32(offset), hi32(offset)) and key (lo32(seed), hi32(seed)), and is kept
 * iff that word >= floor(p * 2^32).  A training loop gives each step and
 * layer its own (seed, offset).
 * keep: uint32 [m, k/32], bit j % 32 of word i * (k/32) + j / 32 set iff
 * element (i, j) is kept.  x_drop: bf16 [m, k] = x * keep (bit-exact: the
 * kept bits of x, +0 elsewhere); the 1 / (1 - p) is applied by the layer
 * calls in the LoRA scale, s_d = fl32(s / (1 - p)).
 * p: fp32 in [0, 1) (QN_ERR_ARG otherwise). */

/* The mask and x_drop alone.  k % 32 == 0 (QN_ERR_SHAPE otherwise). */
qn_status lora_dropout(const void* x, int64_t m, int64_t k, float p, uint64_t seed, uint64_t offset,
                       void* x_drop, uint32_t* keep, qn_stream_t stream);

/* Workspace for the two dropout layer calls (larger than
 * qlora_workspace_bytes: it also holds dy W_hat in fp32, m * k_in floats). */
size_t qlora_dropout_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int r);

/* Training forward with LoRA dropout (always the tensor-core GEMM path):
 *   x_drop, keep = lora_dropout(x, p, seed, offset)
 *   y = x W_hat^T + s_d (x_drop A^T) B^T
 * u_save: NULL or bf16 [m, r] receiving x_drop A^T (without the 1/(1-p)).
 * x_drop and keep are outputs the backward needs (it does not read x).
 * r > 0; other arguments as for qlora_linear_fwd. */
qn_status qlora_linear_fwd_dropout(const void* x, int64_t m, const qn_nf4_weight* w,
                                   const void* A, const void* B, int r, float alpha,
                                   float p, uint64_t seed, uint64_t offset,
                                   void* y, void* u_save, void* x_drop, uint32_t* keep,
                                   void* ws, size_t ws_bytes, qn_stream_t stream);

/* Backward of qlora_linear_fwd_dropout, from its x_drop, keep (and u_save):
 *   dx = dy W_hat + s_d keep * ((dy B) A)   (bf16; skipped if dx NULL)
 *   dA = s_d (dy B)^T x_drop                (fp32 [r, k_in])
 *   dB = s_d dy^T (x_drop A^T)              (fp32 [n_out, r])
 * dy W_hat is kept in fp32 and dx is rounded to bf16 once.
 * u: NULL (recomputed from x_drop and A) or the forward's u_save.
 * keep may be NULL when dx is NULL. */
qn_status qlora_linear_bwd_dropout(const void* dy, const void* x_drop, const uint32_t* keep, int64_t m,
                                   const qn_nf4_weight* w, const void* A, const void* B,
                                   int r, float alpha, float p, const void* u,
                                   void* dx, float* dA, float* dB,
                                   void* ws, size_t ws_bytes, qn_stream_t stream);

/* ---------------------------------------------------------------- optimizer */

/* One AdamW step on a LoRA matrix (or on all of a model's adapters laid out
 * in one array) with 8-bit states.
 * [skyvanguard lesson, "Optimizadores Paginados": QLoRA trains with
 *  paged_adamw_8bit, Adam with 8-bit states; "Cálculo de Memoria": the
 *  8-bit optimizer needs a fraction of fp32 Adam's 8 bytes per parameter.
 *  "Módulo 4: QLoRA", 4.4: only the LoRA matrices train.  Paging (moving
 *  states to host memory) is not provided.]
 * The pages fix no state format; this library's: m and v in blocks of 256
 * consecutive values, each block one fp32 scale (absmax / 448) and one FP8
 * E4M3 code per value (value * (448 / absmax), or value / scale where that
 * reciprocal overflows fp32; round to nearest even, saturating; zero stored
 * as +0).  Zero codes and zero scales are the
 * initial state.  The step, in fp32, one IEEE operation at a time
 * (constants formed in fp64 from the fp32 arguments and rounded once):
 *   m = b1 m0 + (1 - b1) g,  v = b2 v0 + (1 - b2) g g,
 *   p = p (1 - lr wd) - (lr / (1 - b1^t)) (m / (sqrt(v) / sqrt(1 - b2^t) + eps)),
 * the division by sqrt(1 - b2^t) as a product with its fp32 reciprocal;
 * then m and v are re-encoded.
 * param: fp32 [n] master values, updated in place; grad: fp32 [n];
 * m_codes, v_codes: uint8 [n]; m_scale, v_scale: fp32 [qlora_adamw8_blocks(n)];
 * param_bf16: NULL or bf16 [n], receives bf16(param) (the copy the layer
 * reads).  All DEVICE, caller-owned, 16-byte aligned.  step t >= 1;
 * 0 <= beta < 1; eps > 0; lr, weight_decay >= 0 (QN_ERR_ARG otherwise). */
size_t qlora_adamw8_blocks(int64_t n);
qn_status qlora_adamw8_step(float* param, const float* grad, int64_t n,
                            uint8_t* m_codes, float* m_scale, uint8_t* v_codes, float* v_scale,
                            void* param_bf16, float lr, float beta1, float beta2, float eps,
                            float weight_decay, int64_t step, qn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
