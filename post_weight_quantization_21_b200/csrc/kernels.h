// Internal launchers of the GPTQ solver kernels (host side; not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gptq.h"

namespace gptq {

// A1, fp32 FMA path (any input dtype; the product path for fp32 inputs)
size_t hessian_simt_workspace(int64_t n_tokens, int64_t d);
gptq_status hessian_simt_launch(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d, float* H,
                                float scale, int32_t accumulate, void* workspace, cudaStream_t stream);

// A1, tcgen05 tensor-core path for 16-bit inputs
bool hessian_tc_supported(int64_t n_tokens, int64_t d, int32_t x_dtype);
size_t hessian_tc_workspace(int64_t n_tokens, int64_t d);
int hessian_tc_launches(int64_t n_tokens, int64_t d);
gptq_status hessian_tc_launch(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d, float* H, float scale,
                              int32_t accumulate, int32_t* status, void* workspace, cudaStream_t stream);

// fp32-accurate 128x128-tile products on the tensor cores (3xTF32), gemm_tf32x3.cu
enum Tf32x3Kind { kGemmTrsm = 0, kGemmSyrk = 1, kGemmTrtriT = 2, kGemmTrtriY = 3, kGemmLazy = 4 };
enum Tf32x3Epi { kEpiStore = 0, kEpiStoreNeg = 1, kEpiSub = 2, kEpiStoreT = 3 };
struct Tf32x3Args {
  int kind, epi, b_mn, tiles;  // what, epilogue, B operand MN-major, work units
  int p, skip;                 // trsm / syrk: panel; syrk: leading output tiles left out
  int g, D;                    // trtri levels: half size and count of 128-blocks
  int i1, i2, k, tiles_n;      // lazy update: U rows [i1, i1 + k), output columns from i2, column tiles
  int o_w, o_h;                // output extent (columns, rows)
  uint32_t idesc;              // set by the launcher
  int32_t* status;
};
// 2-D fp32 tensor map (rows x cols, row stride ld elements), boxes of 32 columns x box_rows rows,
// 128-byte swizzle (32-byte granules for an MN-major operand); false when the base or the stride is
// not 16-byte aligned
bool tf32x3_map(CUtensorMap* map, const float* base, int64_t rows, int64_t cols, int64_t ld, int box_rows,
                bool mn_operand = false);
// A: box rows 128 (K-major); B: box rows 128 (K-major) or 32 (MN-major map); O: box rows 32
gptq_status tf32x3_gemm_launch(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& O, Tf32x3Args a,
                               cudaStream_t stream, int reserve_sms = 0);

// fp32-accurate C -= A B^T on CTA pairs with operands split into tf32 hi / lo beforehand
// (gemm_tf32x3_pair.cu).  A and B are [rows, 128] K-major panels; C is reduce-added through `out`.
enum PairKind { kPairSyrk = 0, kPairLazy = 1 };
struct PairGemmArgs {
  int kind, tiles;
  int tiles_n;          // lazy: 256-column tiles
  int super_r, super_c; // syrk: 256-row and 256-column super-blocks of the updated region (R >= C)
  int cols_blk;         // syrk: 128-block columns of the region (a super-block may reach past them)
  int row0;             // first row of A and of B in the operand maps for super-block 0
  int nk;               // K stages of 32
  int o_w, o_h;         // output extent (columns, rows)
  int out_y0, out_x0;   // output origin of tile (0, 0)
  int skip_diag;        // syrk: leave the first diagonal 128-block to the look-ahead
  uint32_t idesc;       // set by the launcher
  int32_t* status;
};
// [rows, cols] hi or lo operand (row stride ld) for the pair GEMM
bool split_map(CUtensorMap* map, const float* base, int64_t rows, int64_t cols, int64_t ld);
// rows x 128 panel (row stride ld) -> hi / lo (row stride dld)
gptq_status split_rows_launch(const float* src, int64_t ld, int64_t rows, float* hi, float* lo, int64_t dld,
                              cudaStream_t s);
// k_rows x cols panel (row stride ld) -> hi / lo [cols, k_rows] (K-major)
gptq_status split_transpose_launch(const float* src, int64_t ld, int64_t cols, int k_rows, float* hi, float* lo,
                                   cudaStream_t s);
gptq_status tf32x3_pair_launch(const CUtensorMap& a_hi, const CUtensorMap& a_lo, const CUtensorMap& b_hi,
                               const CUtensorMap& b_lo, const CUtensorMap& out, PairGemmArgs g, cudaStream_t s,
                               int reserve_pairs = 0);

// A2 + A3
// with_pair: room for the split panel of the pair-GEMM trailing update (the workspace entry point)
size_t prepare_blocked_workspace(int64_t d, bool with_pair = true);
// lookahead: factor the next diagonal block on a library-owned second stream (made once per device)
gptq_status prepare_blocked_launch(const float* H, int64_t d, float damp, float* U, int32_t* status,
                                   void* workspace, cudaStream_t stream, bool lookahead, bool pair = true);
size_t prepare_workspace(int64_t d);
// the blocked path's tile products run as 3xTF32 tensor-core products; the launch takes exactly this
// path or fails
bool prepare_uses_tensor_cores(int64_t d);
gptq_status prepare_launch(const float* H, int64_t d, float damp, float* U, int32_t* status,
                           void* workspace, cudaStream_t stream, bool lookahead = true, bool pair = true);
// same, with the scratch in a static device array (d <= GPTQ_PREPARE_STATIC_MAX_D)
gptq_status prepare_launch_static(const float* H, int64_t d, float damp, float* U, int32_t* status,
                                  cudaStream_t stream);

// A4 - A6
size_t quantize_workspace(int64_t m, int64_t d, int block_size);
bool quantize_fused(int64_t m, int64_t d);  // one launch per layer (U resident in L2) rather than launches per block
// the lazy block updates run as 3xTF32 tensor-core products (the per-block path without GPTQ_FLAG_FP32_FMA,
// with a tile count that fits 32 bits); the launch takes exactly this path or fails
bool quantize_lazy_on_tensor_cores(int64_t m, int64_t d, uint32_t flags);
// clear_status = false keeps what earlier launches of the same call recorded in the status word
gptq_status quantize_launch(const void* W, int32_t w_dtype, int64_t m, int64_t d, const float* U,
                            const gptq_quant_cfg& cfg, uint8_t* codes, float* scales, int32_t* zeros,
                            int32_t* status, void* workspace, cudaStream_t stream, bool clear_status = true);

// act-order (act_order.cu)
gptq_status act_order_launch(const float* H, int64_t d, int32_t* perm, float* H_perm, int32_t* status,
                             cudaStream_t stream);
size_t quantize_act_order_workspace(int64_t m, int64_t d, int block_size);
gptq_status quantize_act_order_launch(const void* W, int32_t w_dtype, int64_t m, int64_t d, const float* U_perm,
                                      const int32_t* perm, const gptq_quant_cfg& cfg, uint8_t* codes,
                                      float* scales, int32_t* zeros, int32_t* status, void* workspace,
                                      cudaStream_t stream);

// inference with the packed weights (dequant_matmul.cu)
size_t dequant_matmul_workspace(int64_t m, int64_t d, int64_t batch);
gptq_status dequant_matmul_launch(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m,
                                  int64_t d, int32_t bits, int32_t group_size, const void* X, int32_t x_dtype,
                                  int64_t batch, float* Y, int32_t* status, void* workspace, cudaStream_t stream);

gptq_status dequantize_launch(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m, int64_t d,
                              int32_t bits, int32_t group_size, void* out, int32_t out_dtype, cudaStream_t stream);

// A7
gptq_status pack_launch(const uint8_t* codes, int64_t m, int64_t d, int32_t bits, int32_t* packed,
                        cudaStream_t stream);

}  // namespace gptq

namespace gptq {
// A1 dispatcher: tensor cores for 16-bit inputs, fp32 FMA for fp32 inputs.
size_t hessian_workspace(int64_t n_tokens, int64_t d, int32_t x_dtype);
gptq_status hessian_launch(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d, float* H,
                           float scale, int32_t accumulate, int32_t* status, void* workspace,
                           cudaStream_t stream);
}  // namespace gptq
