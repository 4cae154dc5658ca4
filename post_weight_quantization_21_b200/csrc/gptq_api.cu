// The C ABI declared in include/gptq.h: host-side validation, then launches on the caller's stream.
#include <stdio.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

using gptq::aligned;

namespace gptq {
static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace gptq

namespace {

bool valid_dtype(int32_t t) { return t == GPTQ_BF16 || t == GPTQ_FP16 || t == GPTQ_FP32; }
size_t dtype_size(int32_t t) { return t == GPTQ_FP32 ? 4 : 2; }

constexpr int64_t kMaxDim = 1 << 20;  // channel / row limit (keeps every 32-bit tile index in range)

// act_order: whether the caller takes the act-order path (GPTQ_FLAG_ACT_ORDER allowed); the plain
// gptq_quantize_layer has no permutation argument, so the flag is an error there
gptq_status check_cfg(const gptq_quant_cfg* cfg, int64_t d, bool act_order = false) {
  if (cfg == nullptr) return GPTQ_ERR_ARG;
  if (cfg->bits < 2 || cfg->bits > 4) return GPTQ_ERR_ARG;
  if (cfg->block_size != 32 && cfg->block_size != 64 && cfg->block_size != 128) return GPTQ_ERR_ARG;
  if ((cfg->flags & GPTQ_FLAG_ACT_ORDER) && !act_order) return GPTQ_ERR_ARG;
  if (cfg->flags & ~(GPTQ_FLAG_ACT_ORDER | GPTQ_FLAG_FP32_FMA)) return GPTQ_ERR_ARG;
  if (d % cfg->block_size) return GPTQ_ERR_ARG;
  const int g = cfg->group_size;
  if (g < 0) return GPTQ_ERR_ARG;
  if (g) {
    if (g % 32 || d % g) return GPTQ_ERR_ARG;
    if (g % cfg->block_size && cfg->block_size % g) return GPTQ_ERR_ARG;
  }
  return GPTQ_OK;
}

}  // namespace

extern "C" {

int32_t gptq_abi_version(void) { return GPTQ_ABI_VERSION; }

uint64_t gptq_kernel_launches(void) { return gptq::g_launches.load(std::memory_order_relaxed); }

int32_t gptq_tensor_core_phases(int64_t m, int64_t d, int64_t n_tokens, int32_t x_dtype, const gptq_quant_cfg* cfg) {
  if (m <= 0 || d <= 0 || n_tokens < 0 || d > kMaxDim || !valid_dtype(x_dtype) || check_cfg(cfg, d, true) != GPTQ_OK)
    return -1;
  int32_t mask = 0;
  if (gptq::hessian_tc_supported(n_tokens, d, x_dtype)) mask |= GPTQ_TC_HESSIAN;
  if (gptq::prepare_uses_tensor_cores(d)) mask |= GPTQ_TC_PREPARE;
  if (gptq::quantize_lazy_on_tensor_cores(m, d, cfg->flags)) mask |= GPTQ_TC_LAZY;
  return mask;
}

const char* gptq_status_string(int32_t status) {
  switch (status) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_ARG: return "invalid argument";
    case GPTQ_ERR_UNSUPPORTED: return "unsupported option";
    case GPTQ_ERR_NOT_PD: return "dampened Hessian is not positive definite";
    case GPTQ_ERR_CUDA: return "CUDA error";
    case GPTQ_ERR_TIMEOUT: return "bounded device wait gave up";
    case GPTQ_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

size_t gptq_hessian_workspace_size(int64_t n_tokens, int64_t d, int32_t x_dtype) {
  if (n_tokens < 0 || d <= 0 || d > kMaxDim || !valid_dtype(x_dtype)) return 0;
  return gptq::hessian_workspace(n_tokens, d, x_dtype);
}

gptq_status gptq_hessian_accumulate(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d, float* H,
                                    float scale, int32_t accumulate, int32_t* dev_status, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!valid_dtype(x_dtype) || n_tokens < 0 || d <= 0 || d > kMaxDim || d % 8) return GPTQ_ERR_ARG;
  if (H == nullptr || dev_status == nullptr || (n_tokens > 0 && X == nullptr)) return GPTQ_ERR_ARG;
  if (!aligned(X, 16) || !aligned(H, 16) || !aligned(dev_status, 4)) return GPTQ_ERR_ARG;
  if (accumulate != 0 && accumulate != 1) return GPTQ_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t need = n_tokens ? gptq::hessian_workspace(n_tokens, d, x_dtype) : 0;
  if (need && (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)))
    return GPTQ_ERR_WORKSPACE;
  // a fresh sum starts with a clear status word; accumulating calls keep what earlier calls recorded
  if (!accumulate) GPTQ_CUDA_TRY(cudaMemsetAsync(dev_status, 0, 2 * sizeof(int32_t), s));
  if (n_tokens == 0) {
    if (!accumulate) GPTQ_CUDA_TRY(cudaMemsetAsync(H, 0, (size_t)d * d * sizeof(float), s));
    return GPTQ_OK;
  }
  return gptq::hessian_launch(X, x_dtype, n_tokens, d, H, scale, accumulate, dev_status, workspace, s);
}

size_t gptq_prepare_workspace_size(int64_t d) {
  if (d <= 0 || d > kMaxDim) return 0;
  return gptq::prepare_workspace(d);
}

gptq_status gptq_prepare_uinv(const float* H, int64_t d, float damp, float* U, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (d <= 0 || d > kMaxDim || H == nullptr || U == nullptr || dev_status == nullptr) return GPTQ_ERR_ARG;
  if (!(damp >= 0.0f) || !aligned(H, 16) || !aligned(U, 16) || !aligned(dev_status, 4)) return GPTQ_ERR_ARG;
  if ((const void*)H == (const void*)U) return GPTQ_ERR_ARG;
  const size_t need = gptq::prepare_workspace(d);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return GPTQ_ERR_WORKSPACE;
  return gptq::prepare_launch(H, d, damp, U, dev_status, workspace, static_cast<cudaStream_t>(stream));
}

gptq_status gptq_prepare_uinv_static(const float* H, int64_t d, float damp, float* U, int32_t* dev_status,
                                     void* stream) {
  if (d <= 0 || H == nullptr || U == nullptr || dev_status == nullptr) return GPTQ_ERR_ARG;
  if (!(damp >= 0.0f) || !aligned(H, 16) || !aligned(U, 16) || !aligned(dev_status, 4)) return GPTQ_ERR_ARG;
  if ((const void*)H == (const void*)U) return GPTQ_ERR_ARG;
  if (d > GPTQ_PREPARE_STATIC_MAX_D) return GPTQ_ERR_WORKSPACE;
  return gptq::prepare_launch_static(H, d, damp, U, dev_status, static_cast<cudaStream_t>(stream));
}

size_t gptq_quantize_workspace_size(int64_t m, int64_t d, const gptq_quant_cfg* cfg) {
  if (m <= 0 || d <= 0 || d > kMaxDim || m > kMaxDim * 64 || cfg == nullptr) return 0;
  if (check_cfg(cfg, d) != GPTQ_OK) return 0;
  return gptq::quantize_workspace(m, d, cfg->block_size);
}

gptq_status gptq_quantize_layer(const void* W, int32_t w_dtype, int64_t m, int64_t d, const float* U,
                                const gptq_quant_cfg* cfg, uint8_t* codes, float* scales, int32_t* zeros,
                                int32_t* dev_status, void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_dtype(w_dtype) || m <= 0 || d <= 0 || d > kMaxDim || m > kMaxDim * 64 || d % 32)
    return GPTQ_ERR_ARG;
  gptq_status st = check_cfg(cfg, d);
  if (st != GPTQ_OK) return st;
  if (!W || !U || !codes || !scales || !zeros || !dev_status) return GPTQ_ERR_ARG;
  if (!aligned(W, dtype_size(w_dtype)) || !aligned(U, 16) || !aligned(codes, 4) || !aligned(scales, 4) ||
      !aligned(zeros, 4) || !aligned(dev_status, 4))
    return GPTQ_ERR_ARG;
  const size_t need = gptq::quantize_workspace(m, d, cfg->block_size);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return GPTQ_ERR_WORKSPACE;
  return gptq::quantize_launch(W, w_dtype, m, d, U, *cfg, codes, scales, zeros, dev_status, workspace,
                               static_cast<cudaStream_t>(stream));
}

gptq_status gptq_act_order(const float* H, int64_t d, int32_t* perm, float* H_perm, int32_t* dev_status,
                           void* stream) {
  if (d <= 0 || d > kMaxDim || H == nullptr || perm == nullptr || H_perm == nullptr || dev_status == nullptr)
    return GPTQ_ERR_ARG;
  if (!aligned(H, 4) || !aligned(perm, 4) || !aligned(H_perm, 4) || !aligned(dev_status, 4)) return GPTQ_ERR_ARG;
  if ((const void*)H == (const void*)H_perm) return GPTQ_ERR_ARG;
  return gptq::act_order_launch(H, d, perm, H_perm, dev_status, static_cast<cudaStream_t>(stream));
}

size_t gptq_quantize_act_order_workspace_size(int64_t m, int64_t d, const gptq_quant_cfg* cfg) {
  if (m <= 0 || d <= 0 || d > kMaxDim || m > kMaxDim * 64 || cfg == nullptr) return 0;
  if (check_cfg(cfg, d, true) != GPTQ_OK) return 0;
  return gptq::quantize_act_order_workspace(m, d, cfg->block_size);
}

gptq_status gptq_quantize_layer_act_order(const void* W, int32_t w_dtype, int64_t m, int64_t d, const float* U_perm,
                                          const int32_t* perm, const gptq_quant_cfg* cfg, uint8_t* codes,
                                          float* scales, int32_t* zeros, int32_t* dev_status, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  if (!valid_dtype(w_dtype) || m <= 0 || d <= 0 || d > kMaxDim || m > kMaxDim * 64 || d % 32)
    return GPTQ_ERR_ARG;
  gptq_status st = check_cfg(cfg, d, true);
  if (st != GPTQ_OK) return st;
  if (!W || !U_perm || !perm || !codes || !scales || !zeros || !dev_status) return GPTQ_ERR_ARG;
  if (!aligned(W, dtype_size(w_dtype)) || !aligned(U_perm, 16) || !aligned(perm, 4) || !aligned(codes, 4) ||
      !aligned(scales, 4) || !aligned(zeros, 4) || !aligned(dev_status, 4))
    return GPTQ_ERR_ARG;
  const size_t need = gptq::quantize_act_order_workspace(m, d, cfg->block_size);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return GPTQ_ERR_WORKSPACE;
  return gptq::quantize_act_order_launch(W, w_dtype, m, d, U_perm, perm, *cfg, codes, scales, zeros, dev_status,
                                         workspace, static_cast<cudaStream_t>(stream));
}

gptq_status gptq_pack(const uint8_t* codes, int64_t m, int64_t d, int32_t bits, int32_t* packed, void* stream) {
  if (m <= 0 || d <= 0 || d % 32 || bits < 2 || bits > 4 || !codes || !packed) return GPTQ_ERR_ARG;
  if (!aligned(packed, 4)) return GPTQ_ERR_ARG;
  if (m > kMaxDim * 64 || d > kMaxDim) return GPTQ_ERR_ARG;
  return gptq::pack_launch(codes, m, d, bits, packed, static_cast<cudaStream_t>(stream));
}

size_t gptq_dequant_matmul_workspace_size(int64_t m, int64_t d, int64_t batch) {
  if (m <= 0 || d <= 0 || d > kMaxDim || m > kMaxDim * 64 || batch <= 0) return 0;
  return gptq::dequant_matmul_workspace(m, d, batch);
}

gptq_status gptq_dequant_matmul(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m,
                                int64_t d, int32_t bits, int32_t group_size, const void* X, int32_t x_dtype,
                                int64_t batch, float* Y, int32_t* dev_status, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (m <= 0 || d <= 0 || d % 32 || d > kMaxDim || m > (int64_t)0x7fffffff - 64 || bits < 2 || bits > 4)
    return GPTQ_ERR_ARG;
  if (batch <= 0 || batch > 1024 || !valid_dtype(x_dtype)) return GPTQ_ERR_ARG;
  if (group_size < 0 || (group_size && (group_size % 32 || d % group_size))) return GPTQ_ERR_ARG;
  if (!packed || !scales || !zeros || !X || !Y || !dev_status) return GPTQ_ERR_ARG;
  // packed rows start on 16-byte boundaries when d % 128 == 0 (the bulk-copied form needs it)
  if (!aligned(packed, 16) || !aligned(scales, 4) || !aligned(zeros, 4) || !aligned(X, 16) || !aligned(Y, 4) ||
      !aligned(dev_status, 4))
    return GPTQ_ERR_ARG;
  const size_t need = gptq::dequant_matmul_workspace(m, d, batch);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return GPTQ_ERR_WORKSPACE;
  return gptq::dequant_matmul_launch(packed, scales, zeros, m, d, bits, group_size, X, x_dtype, batch, Y, dev_status,
                                     workspace, static_cast<cudaStream_t>(stream));
}

gptq_status gptq_dequantize(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m, int64_t d,
                            int32_t bits, int32_t group_size, void* W_hat, int32_t out_dtype, void* stream) {
  if (m <= 0 || d <= 0 || d % 32 || d > kMaxDim || m > kMaxDim * 64 || bits < 2 || bits > 4) return GPTQ_ERR_ARG;
  if (!valid_dtype(out_dtype)) return GPTQ_ERR_ARG;
  if (group_size < 0 || (group_size && (group_size % 32 || d % group_size))) return GPTQ_ERR_ARG;
  if (!packed || !scales || !zeros || !W_hat) return GPTQ_ERR_ARG;
  if (!aligned(packed, 4) || !aligned(scales, 4) || !aligned(zeros, 4) || !aligned(W_hat, dtype_size(out_dtype)))
    return GPTQ_ERR_ARG;
  return gptq::dequantize_launch(packed, scales, zeros, m, d, bits, group_size, W_hat, out_dtype,
                                 static_cast<cudaStream_t>(stream));
}

gptq_status gptq_read_status(const int32_t* dev_status, void* stream, int64_t* detail) {
  if (dev_status == nullptr) return GPTQ_ERR_ARG;
  int32_t h[2] = {0, 0};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(h, dev_status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (detail) *detail = h[1];
  return static_cast<gptq_status>(h[0]);
}

}  // extern "C"
