/*
 * gptq.h — C ABI of the GPTQ layer-wise quantization solver for NVIDIA B200 (sm_100a).
 *
 * GPTQ (Frantar, Ashkboos, Hoefler, Alistarh; ICLR 2023) quantizes one linear layer W[out, in] at a
 * time so that the layer's output on calibration inputs X[tokens, in] changes as little as possible
 * (FDE Interviews breakdown of GPTQ, section 01 "The paper in one minute"; zhiliyouxian blog
 * "GPTQ：用于生成式预训练 Transformer 的准确训练后量化", section 数学基础 and the layer routine in
 * 算法流程, whose arguments are W [out_features, in_features], X [batch, in_features], bits).
 *
 * The solver runs in four calls, in this order:
 *   1. gptq_hessian_accumulate   H  = 2 X^T X                      (A1)
 *   2. gptq_prepare_uinv         Hd = H + damp*mean(diag H)*I;  U = chol(Hd^-1), upper   (A2, A3)
 *   3. gptq_quantize_layer       column loop + lazy block updates -> codes, scales, zeros (A4-A6)
 *   4. gptq_pack                 b-bit codes -> int32 words                                (A7)
 *
 * Conventions shared by every entry point:
 *  - Matrices are dense and row-major with no padding (leading dimension = number of columns).
 *  - Every pointer argument except `cfg` and `detail` is DEVICE memory on the current CUDA device,
 *    allocated and owned by the caller.  The library allocates no device or host memory and keeps no
 *    state between calls (apart from a cached driver entry point).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only enqueues work on
 *    that stream and returns; results are ready when the stream reaches that point.
 *  - Arguments are validated on the host before anything is enqueued; a bad argument returns
 *    GPTQ_ERR_ARG (or GPTQ_ERR_UNSUPPORTED / GPTQ_ERR_WORKSPACE) and enqueues nothing.
 *  - Failures found on the device (a non-positive pivot, a bounded wait that gave up) are written
 *    to the caller's device status word `dev_status` (int32[2]: code, detail), never trapped; read it
 *    with gptq_read_status.  Kernels never spin without an iteration limit.
 *  - A launch failure returns GPTQ_ERR_CUDA.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPTQ_ABI_VERSION 2

#if defined(__GNUC__)
#define GPTQ_API __attribute__((visibility("default")))
#else
#define GPTQ_API
#endif

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_ARG = 1,          /* null pointer, bad size, misaligned pointer, bad combination    */
  GPTQ_ERR_UNSUPPORTED = 2,  /* a valid option this library does not implement                */
  GPTQ_ERR_NOT_PD = 3,       /* device: the dampened Hessian is not positive definite          */
  GPTQ_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed                           */
  GPTQ_ERR_TIMEOUT = 5,      /* device: a bounded wait inside a kernel gave up                 */
  GPTQ_ERR_WORKSPACE = 6     /* workspace pointer null or smaller than the *_workspace_size    */
} gptq_status;

typedef enum { GPTQ_BF16 = 0, GPTQ_FP16 = 1, GPTQ_FP32 = 2 } gptq_dtype;

/* Flags of gptq_quant_cfg.flags. */
#define GPTQ_FLAG_ACT_ORDER 1u /* columns in descending diag(H) order ("desc_act"): only with
                                  gptq_quantize_layer_act_order, which takes the permutation; an
                                  error (GPTQ_ERR_ARG) in gptq_quantize_layer */
#define GPTQ_FLAG_FP32_FMA 2u  /* lazy block updates on the fp32 FMA units instead of the tensor cores
                                  (3xTF32: tf32 hi/lo splits of both operands, fp32 accumulation) */

/* Quantization settings of one layer (zhiliyouxian blog, 实践指南: bits, group_size, desc_act;
 * agent.csdn.net "GPTQ量化参数搜索工具", 关键参数说明 table: bits, group_size, zero point;
 * FDE breakdown figure step 4: blocks of 128 columns). */
typedef struct {
  int32_t bits;        /* 2, 3 or 4: codes lie in [0, 2^bits - 1]                                 */
  int32_t group_size;  /* 0: one grid per row; else a multiple of 32 that divides d, and either
                          group_size divides block_size or block_size divides group_size         */
  int32_t block_size;  /* columns per lazy-update block: 32, 64 or 128                            */
  uint32_t flags;      /* GPTQ_FLAG_* ; 0 for the plain method                                    */
} gptq_quant_cfg;

/* ------------------------------------------------------------------------------------------
 * A1  H = accumulate ? H + scale * X^T X : scale * X^T X
 *
 * The curvature of the layer-wise least-squares objective, H = 2 X X^T with X as [in, tokens]
 * (FDE breakdown, section 01 and figure "THE IDEA, VISUALLY"); here X is [tokens, in] so H = 2 X^T X
 * and `scale` = 2 reproduces the pages.  The sum over tokens is additive, so a caller may feed the
 * calibration set in chunks with accumulate = 1.
 *
 *   X          [n_tokens, d] row-major, dtype x_dtype (BF16 / FP16 use the tensor cores with fp32
 *              accumulation; FP32 uses fp32 FMA).  Must be 16-byte aligned.
 *   H          [d, d] fp32 row-major.  On return the upper triangle (j >= i) holds the result; the
 *              strict lower triangle is left unspecified.
 *   workspace  >= gptq_hessian_workspace_size(n_tokens, d, x_dtype) bytes, 256-byte aligned.
 *   dev_status int32[2] device status word: cleared at the start of a call with accumulate = 0 (a
 *              chunked sequence keeps the first failure of any of its calls); GPTQ_ERR_TIMEOUT if a
 *              bounded device wait gave up.
 *   Requires d % 8 == 0, n_tokens >= 0 (0 tokens gives H = 0 or leaves H unchanged).
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_hessian_accumulate(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d,
                                    float* H, float scale, int32_t accumulate, int32_t* dev_status,
                                    void* workspace, size_t workspace_bytes, void* stream);
GPTQ_API size_t gptq_hessian_workspace_size(int64_t n_tokens, int64_t d, int32_t x_dtype);

/* ------------------------------------------------------------------------------------------
 * A2 + A3  U = upper Cholesky factor of (H + damp * mean(diag H) * I)^-1
 *
 * Dampening: zhiliyouxian blog 算法流程 ("H = H + lambda * I") and 实践指南 (damp_percent = 0.01);
 * nubint.ai review, "Proposed method" (Cholesky reformulation and dampening for stability).
 * U: FDE breakdown figure step 2 ("U = chol(H^-1)") and section 01 (rows of the inverse Hessian
 * from a Cholesky decomposition).  U^T U = Hd^-1, U upper with positive diagonal.
 *
 *   H          [d, d] fp32, upper triangle read (as written by gptq_hessian_accumulate); unchanged.
 *   U          [d, d] fp32 output: upper triangle = the factor, strict lower triangle = 0.
 *              Also used as scratch during the call; must not alias H.
 *   dev_status int32[2]: cleared at the start of the call; {GPTQ_ERR_NOT_PD, pivot column} if the
 *              dampened matrix is not positive definite (U is then unspecified); GPTQ_ERR_TIMEOUT
 *              if a bounded device wait gave up.
 *   workspace  >= gptq_prepare_workspace_size(d) bytes, 256-byte aligned.
 *   d <= 1024 runs as one cooperative launch.  Larger orders run a blocked factorisation whose block
 *   products use the tensor cores as 3xTF32 when d % 4 == 0 (fp32 FMA tiles otherwise); their next
 *   diagonal block is factored on a second stream that the library creates once per device (with
 *   two events) and joins back into `stream` before the call's last launch, so the whole call is
 *   ordered on `stream` for the caller.
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_prepare_uinv(const float* H, int64_t d, float damp, float* U, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, void* stream);
GPTQ_API size_t gptq_prepare_workspace_size(int64_t d);

/* ------------------------------------------------------------------------------------------
 * gptq_prepare_uinv_static: the same computation as gptq_prepare_uinv without a workspace argument.
 *
 * The GPTQ pages have no counterpart for this call; it exists for callers that cannot allocate
 * device memory themselves, for example a plugin whose host application owns all device memory
 * through its own pool, or a latency-bound path where no allocator may be called.  The scratch the
 * computation needs (about 4 MiB) is a fixed array compiled into this library; every GPU that loads
 * the library holds it until the process exits.
 *
 *   H, d, damp, U, dev_status, stream: as for gptq_prepare_uinv (U is still caller memory).
 *   d > GPTQ_PREPARE_STATIC_MAX_D returns GPTQ_ERR_WORKSPACE and enqueues nothing.
 *   The first call on each device looks up the array's device address (a host-side runtime call,
 *   with that device current); make that first call before any stream capture.  The address is
 *   cached with the id of the device's context and looked up again when the context changes (after
 *   cudaDeviceReset, say): make the first call after such a change before any stream capture too.
 *   All calls share the one array and it keeps the last call's contents (each call clears the parts
 *   that must start at zero).  Calls that overlap on the GPU, on any streams, race on it: order them.
 *   It creates no CUDA objects: above d = 1024 every launch goes to `stream` (no look-ahead stream).
 *   No memory is allocated or freed.
 * ------------------------------------------------------------------------------------------ */
#define GPTQ_PREPARE_STATIC_MAX_D 8192
GPTQ_API gptq_status gptq_prepare_uinv_static(const float* H, int64_t d, float damp, float* U,
                                              int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------------------------
 * A4 - A6  Column loop with error compensation and lazy block updates.
 *
 * For each column i in natural order (FDE breakdown figure steps 1-4): q_i = clamp(rint(w_i/scale)
 * + zero, 0, 2^b-1); err = (w_i - scale*(q_i - zero)) / U_ii; W[:, j] -= err * U[i, j] for the
 * remaining columns j of the block at once, and for the columns after the block once per block.
 * Grid: asymmetric min/max over the row (per-row, from the original W) or over the group's current
 * values when the loop reaches the group (per-group), the range widened to contain 0.  The scale and
 * the zero point are IEEE fp32 divisions, rounded half-to-even for the zero point.  Each code's
 * quotient w_i / scale is formed as the fp32 product of w_i and the IEEE fp32 reciprocal of the scale,
 * then rounded half-to-even; it differs from the IEEE quotient by about one ulp at most, so a code can
 * be one level away from the division's only when the quotient is within a few ulps of a half-integer.
 *
 *   W          [m, d] row-major, dtype w_dtype (FP16, BF16 or FP32); read only.
 *   U          [d, d] fp32 upper factor from gptq_prepare_uinv (strict lower part ignored).
 *   codes      [m, d] uint8 output, one code per weight.
 *   scales     [m, n_groups] fp32 output, n_groups = group_size ? d / group_size : 1.
 *   zeros      [m, n_groups] int32 output.
 *   dev_status device int32[2]: cleared at the start of the call; a kernel that gives up a bounded
 *              wait records GPTQ_ERR_TIMEOUT there (read with gptq_read_status).
 *   workspace  >= gptq_quantize_workspace_size(m, d, cfg) bytes, 256-byte aligned (holds the
 *              working copy of W in fp32 and the per-block errors).
 *   Requires d % 32 == 0, d % block_size == 0 and `codes` 4-byte aligned.  flags &
 *   GPTQ_FLAG_ACT_ORDER -> GPTQ_ERR_ARG (act-order takes gptq_quantize_layer_act_order).
 *   The lazy block updates run on the tensor cores as 3xTF32 products (each operand split into a
 *   tf32 high part and a tf32 remainder, three MMAs per product, fp32 accumulation: about the
 *   accuracy of fp32 FMA); flags & GPTQ_FLAG_FP32_FMA selects fp32 FMA units instead.
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_quantize_layer(const void* W, int32_t w_dtype, int64_t m, int64_t d,
                                const float* U, const gptq_quant_cfg* cfg, uint8_t* codes,
                                float* scales, int32_t* zeros, int32_t* dev_status, void* workspace,
                                size_t workspace_bytes, void* stream);
GPTQ_API size_t gptq_quantize_workspace_size(int64_t m, int64_t d, const gptq_quant_cfg* cfg);

/* ------------------------------------------------------------------------------------------
 * Act-order ("desc_act": zhiliyouxian blog, 实践指南, off by default there; agent.csdn.net
 * "GPTQ量化参数搜索工具", 关键参数说明).  The pages name the option without defining the order beyond
 * "sort by activation"; here the columns are quantized in descending order of diag(H), ties by column
 * index.  The method is unchanged on the permuted problem H -> P H P^T, W -> W P^T:
 *   gptq_act_order(H) -> perm, H_perm;  gptq_prepare_uinv(H_perm) -> U_perm;
 *   gptq_quantize_layer_act_order(W, U_perm, perm) -> codes in the original column order.
 *
 * gptq_act_order
 *   H          [d, d] fp32, upper triangle read (as written by gptq_hessian_accumulate).
 *   perm       int32 [d] output: perm[i] = the original column quantized at step i.
 *   H_perm     [d, d] fp32 output: upper triangle of P H P^T, H_perm[i][j] = H[perm[i]][perm[j]]
 *              (j >= i); strict lower triangle unspecified.  Must not alias H.  Its first d words
 *              also serve as scratch during the call.
 *   dev_status int32[2]: cleared at the start of the call.  NaN diagonal entries have an
 *              unspecified place in the order.
 *
 * gptq_quantize_layer_act_order: gptq_quantize_layer on W P^T with U_perm, codes returned in the
 * original column order.
 *   W          [m, d] in the ORIGINAL column order (as for gptq_quantize_layer).
 *   U_perm     [d, d] upper factor of the permuted dampened Hessian (gptq_prepare_uinv of H_perm).
 *   perm       int32 [d]: a permutation of 0..d-1 (from gptq_act_order, or the caller's own order).
 *              An entry out of range or repeated is reported on the device as {GPTQ_ERR_ARG, step}
 *              and its columns read as zeros (no access out of bounds).
 *   codes      [m, d] uint8 output in the original column order (4-byte aligned).
 *   scales, zeros  [m, n_groups]: group k is steps k*group_size .. (k+1)*group_size - 1 of the
 *              quantization order, i.e. original columns perm[k*g .. (k+1)*g - 1]; the group of
 *              original column j is (the step at which j is quantized) / group_size.
 *   workspace  >= gptq_quantize_act_order_workspace_size(m, d, cfg) bytes, 256-byte aligned.
 *   cfg->flags may include GPTQ_FLAG_ACT_ORDER or not; GPTQ_FLAG_FP32_FMA applies as usual.
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_act_order(const float* H, int64_t d, int32_t* perm, float* H_perm,
                                    int32_t* dev_status, void* stream);
GPTQ_API gptq_status gptq_quantize_layer_act_order(const void* W, int32_t w_dtype, int64_t m, int64_t d,
                                                   const float* U_perm, const int32_t* perm,
                                                   const gptq_quant_cfg* cfg, uint8_t* codes, float* scales,
                                                   int32_t* zeros, int32_t* dev_status, void* workspace,
                                                   size_t workspace_bytes, void* stream);
GPTQ_API size_t gptq_quantize_act_order_workspace_size(int64_t m, int64_t d, const gptq_quant_cfg* cfg);

/* ------------------------------------------------------------------------------------------
 * A7  Pack b-bit codes into int32 words (storage of 3-/4-bit weights for the inference kernel;
 * FDE breakdown figure, "3-bit weights 66 GB").  Layout: per row a little-endian bit stream, code j
 * in bits [j*b, (j+1)*b), word k = stream bits [32k, 32k+32).  Row stride = d*bits/32 words.
 *
 *   codes      [m, d] uint8, each < 2^bits (higher bits are masked off).
 *   packed     [m, d*bits/32] int32 output.  Requires d % 32 == 0, bits in {2, 3, 4}.
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_pack(const uint8_t* codes, int64_t m, int64_t d, int32_t bits, int32_t* packed,
                      void* stream);

/* ------------------------------------------------------------------------------------------
 * Inference with the packed weights: Y = X @ What^T with What[r, j] = scale[r, g(j)] * (q[r, j] -
 * zero[r, g(j)]), g(j) = j / group_size (0 per-row), q read from the packed words (FDE breakdown,
 * section 01, last paragraph: kernels that read the 3-bit weights and dequantize them on the fly).
 * For a few input rows (batch): every packed word is read once from HBM.
 *
 *   packed     [m, d*bits/32] int32 from gptq_pack; scales / zeros [m, n_groups] from
 *              gptq_quantize_layer.  Under act-order the groups follow the quantization order: pass
 *              the codes in that order (codes[:, perm] packed) and X with its columns permuted alike.
 *   X          [batch, d] row-major, BF16 / FP16 / FP32, 16-byte aligned, |x| < 2^100 (inputs are
 *              pre-scaled by powers of two up to 2^23 inside the kernel).  1 <= batch <= 1024
 *              (processed four rows at a time).  Every product q x is formed exactly and rounded
 *              once; the sums are fp32.
 *   Y          [batch, m] fp32 output.
 *   dev_status int32[2]: cleared at the start of the call; GPTQ_ERR_TIMEOUT if a bounded wait for the
 *              staged copies of the packed words gave up (d % 128 == 0 stages them in shared memory).
 *   workspace  >= gptq_dequant_matmul_workspace_size(m, d, batch) bytes, 256-byte aligned (partial
 *              sums of the column tiles; the final sum runs in tile order, so results are
 *              deterministic).
 *   Requires d % 32 == 0, bits in {2, 3, 4}, group_size 0 or a multiple of 32 dividing d, `packed`
 *   16-byte aligned.
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_dequant_matmul(const int32_t* packed, const float* scales, const int32_t* zeros,
                                         int64_t m, int64_t d, int32_t bits, int32_t group_size, const void* X,
                                         int32_t x_dtype, int64_t batch, float* Y, int32_t* dev_status,
                                         void* workspace, size_t workspace_bytes, void* stream);
GPTQ_API size_t gptq_dequant_matmul_workspace_size(int64_t m, int64_t d, int64_t batch);

/* ------------------------------------------------------------------------------------------
 * The dequantized weights What[r, j] = scale[r, g(j)] * (q[r, j] - zero[r, g(j)]) as a dense matrix
 * (the values a quantized layer computes with; FDE breakdown section 01 and figure step 1: the
 * weights on the b-bit grid), e.g. for running a quantized block forward to produce the next
 * block's calibration inputs.
 *   packed [m, d*bits/32] int32 (gptq_pack), scales / zeros [m, n_groups]; W_hat [m, d] row-major
 *   in out_dtype (BF16 / FP16 rounded to nearest from the fp32 product, or FP32).
 *   Requires d % 32 == 0, bits in {2, 3, 4}, group_size 0 or a multiple of 32 dividing d.
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_dequantize(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m,
                                     int64_t d, int32_t bits, int32_t group_size, void* W_hat, int32_t out_dtype,
                                     void* stream);

/* ------------------------------------------------------------------------------------------
 * Status helpers.
 * gptq_read_status: synchronizes `stream`, copies the device status word to the host, returns the
 * code it holds (GPTQ_OK if clear) and stores its detail (e.g. the failing pivot) in *detail when
 * detail is not NULL.  Returns GPTQ_ERR_CUDA if the copy fails.
 * ------------------------------------------------------------------------------------------ */
GPTQ_API gptq_status gptq_read_status(const int32_t* dev_status, void* stream, int64_t* detail);
GPTQ_API const char* gptq_status_string(int32_t status);
GPTQ_API int32_t gptq_abi_version(void);

/* Diagnostics: total number of CUDA kernels this library has launched in the process (all devices,
 * all threads).  Host-side counter; reading it does not touch the device. */
GPTQ_API uint64_t gptq_kernel_launches(void);

/* Diagnostics: which phases run their block products on the tensor cores for this shape, as a bit
 * mask (host only, no device access):
 *   GPTQ_TC_HESSIAN  H = scale X^T X with tcgen05 kind::f16 (16-bit X, d >= 256, n_tokens >= 64);
 *                    otherwise fp32 FMA tiles.
 *   GPTQ_TC_PREPARE  the blocked factorisation's trsm / syrk / triangular-inverse tiles as 3xTF32
 *                    (d > 1024 and d % 4 == 0); smaller orders run the one-launch fp32 kernel.
 *   GPTQ_TC_LAZY     the lazy block updates as 3xTF32 (the per-block path: d > 4096 or m > 2048,
 *                    and no GPTQ_FLAG_FP32_FMA); otherwise fp32 FMA.
 * Returns -1 when the arguments are invalid. */
#define GPTQ_TC_HESSIAN 1
#define GPTQ_TC_PREPARE 2
#define GPTQ_TC_LAZY 4
GPTQ_API int32_t gptq_tensor_core_phases(int64_t m, int64_t d, int64_t n_tokens, int32_t x_dtype,
                                         const gptq_quant_cfg* cfg);

/* Failure-detection test hook (no counterpart on the pages).  Makes the NEXT Hessian launch on the
 * tensor-core path (16-bit X, see GPTQ_TC_HESSIAN) exercise its timeout path without any fault: its
 * MMA-issuing thread first waits, for at most `cycles` clock cycles, on a barrier that nothing arrives
 * on, gives up, records {GPTQ_ERR_TIMEOUT, 5} in that call's status word and raises the kernel's abort
 * flag; the other roles leave, the copies already issued land (their waits keep the full bound), TMEM
 * is freed and the kernel returns.  H is then unspecified.  The request is taken by one launch (any
 * thread's); cycles <= 0 cancels it.  Calls made afterwards run normally. */
GPTQ_API void gptq_test_hessian_timeout(int64_t cycles);

#ifdef __cplusplus
}
#endif
#endif /* GPTQ_B200_H */
