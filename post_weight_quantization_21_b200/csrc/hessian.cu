// A1 dispatch: H = scale * X^T X (GPTQ's H = 2 X X^T, FDE Interviews breakdown, section 01).
// 16-bit inputs go to the tcgen05 tensor-core kernel; fp32 inputs (and layers too narrow for a
// 128x256 tile) use the fp32 FMA kernel.
#include "common.cuh"
#include "kernels.h"

namespace gptq {

size_t hessian_workspace(int64_t n_tokens, int64_t d, int32_t x_dtype) {
  if (hessian_tc_supported(n_tokens, d, x_dtype)) return hessian_tc_workspace(n_tokens, d);
  return hessian_simt_workspace(n_tokens, d);
}

gptq_status hessian_launch(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d, float* H,
                           float scale, int32_t accumulate, int32_t* status, void* workspace,
                           cudaStream_t stream) {
  if (hessian_tc_supported(n_tokens, d, x_dtype))
    return hessian_tc_launch(X, x_dtype, n_tokens, d, H, scale, accumulate, status, workspace, stream);
  return hessian_simt_launch(X, x_dtype, n_tokens, d, H, scale, accumulate, workspace, stream);
}

}  // namespace gptq
