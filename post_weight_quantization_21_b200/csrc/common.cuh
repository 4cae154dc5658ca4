// Shared helpers of the GPTQ solver kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gptq.h"

#define GPTQ_CUDA_TRY(expr)                                  \
  do {                                                       \
    cudaError_t e__ = (expr);                                \
    if (e__ != cudaSuccess) return GPTQ_ERR_CUDA;            \
  } while (0)

namespace gptq {
void count_launch();
}
// Called right after every kernel launch: counts it and reports a failed launch.
#define GPTQ_LAUNCH_CHECK()      \
  do {                           \
    gptq::count_launch();        \
    GPTQ_CUDA_TRY(cudaGetLastError()); \
  } while (0)

namespace gptq {

constexpr int kWarp = 32;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Records the first device-side failure in the caller's status word {code, detail}.
__device__ __forceinline__ void report_status(int32_t* status, int32_t code, int32_t detail) {
  if (status == nullptr) return;
  if (atomicCAS(status, 0, code) == 0) status[1] = detail;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Asymmetric min/max grid: the range widened to contain 0, an empty range becomes [-1, 1];
// scale = (hi - lo) / maxq and zero = rint(-lo / scale), both quotients IEEE fp32 divisions (once per
// grid); rscale = IEEE fp32 reciprocal of scale.  The column loops form each code's quotient as the
// IEEE fp32 product x * rscale (not contracted into an FMA) instead of the division x / scale: the two
// differ by at most about one ulp, so a code can differ from the division's by one level only when
// the quotient lies within a few ulps of a half-integer.
// Round to the nearest integer, ties to even, with two fp32 adds on the FMA pipe: adding 1.5 * 2^23
// moves |x| < 2^22 into [2^23, 2^24), where the spacing of floats is 1, so the addition itself rounds.
// Equal to rintf(x) for |x| < 2^22; larger magnitudes come out at least 2^22 - 1 in magnitude, beyond
// any b-bit grid, so a following clamp gives the same result as with rintf.
__device__ __forceinline__ float round_even(float x) {
  const float kShift = 12582912.0f;  // 1.5 * 2^23
  return __fsub_rn(__fadd_rn(x, kShift), kShift);
}

__device__ __forceinline__ void grid_from_range(float mn, float mx, float maxq, float& scale,
                                                float& zero, float& rscale) {
  float lo = fminf(mn, 0.0f);
  float hi = fmaxf(mx, 0.0f);
  if (lo == hi) {
    lo = -1.0f;
    hi = 1.0f;
  }
  scale = __fdiv_rn(hi - lo, maxq);
  rscale = __frcp_rn(scale);
  zero = rintf(__fdiv_rn(-lo, scale));
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace gptq
