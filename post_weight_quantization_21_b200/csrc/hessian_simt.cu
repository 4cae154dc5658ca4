// A1 on the fp32 FMA pipe: H = scale * X^T X for fp32 calibration inputs (and a plain reference
// path for 16-bit inputs).  GPTQ's curvature H = 2 X X^T (FDE Interviews breakdown of GPTQ,
// section 01) with X stored [tokens, in].
//
// Work split: 64x64 tiles of the upper triangle of H x token splits.  Each CTA sums its token
// range in fp32 over 512-token chunks and adds each chunk into fp64 accumulators, then writes an
// fp64 partial tile; a second kernel adds the partials of a tile in split order (deterministic)
// and writes the fp32 result.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kT = 64;         // tile edge
constexpr int kKT = 32;        // tokens staged per step
constexpr int kChunk = 512;    // tokens summed in fp32 before the fp64 flush
constexpr int kMinSplitTokens = 2048;

struct SimtPlan {
  int D;         // tile blocks per dimension
  int tiles;     // upper-triangle tiles
  int splits;    // token splits
  int64_t tokens_per_split;
};

SimtPlan plan(int64_t n_tokens, int64_t d) {
  SimtPlan p;
  p.D = (int)((d + kT - 1) / kT);
  p.tiles = p.D * (p.D + 1) / 2;
  int64_t want = (4 * 148 + p.tiles - 1) / p.tiles;
  int64_t max_by_tokens = (n_tokens + kMinSplitTokens - 1) / kMinSplitTokens;
  int64_t s = want < max_by_tokens ? want : max_by_tokens;
  if (s < 1) s = 1;
  p.splits = (int)s;
  p.tokens_per_split = (n_tokens + s - 1) / s;
  p.tokens_per_split = (p.tokens_per_split + kKT - 1) / kKT * kKT;
  return p;
}

__device__ __forceinline__ void upper_tile(int t, int D, int& bi, int& bj) {
  // row bi holds tiles (bi, bi..D-1)
  int r = 0;
  while (t >= D - r) {
    t -= D - r;
    ++r;
  }
  bi = r;
  bj = r + t;
}

template <typename T>
__global__ void __launch_bounds__(256) hessian_partial_kernel(const T* __restrict__ X, int64_t n_tokens,
                                                             int d, int D, int64_t tokens_per_split,
                                                             double* __restrict__ partial) {
  __shared__ float xa[kKT][kT + 4];
  __shared__ float xb[kKT][kT + 4];
  int bi, bj;
  upper_tile(blockIdx.x, D, bi, bj);
  const int i0 = bi * kT, j0 = bj * kT;
  const int64_t t_begin = (int64_t)blockIdx.y * tokens_per_split;
  int64_t t_end = t_begin + tokens_per_split;
  if (t_end > n_tokens) t_end = n_tokens;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4];
  double acc64[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      acc[a][b] = 0.f;
      acc64[a][b] = 0.0;
    }
  int in_chunk = 0;
  for (int64_t t0 = t_begin; t0 < t_end; t0 += kKT) {
    for (int e = threadIdx.x; e < kKT * kT; e += blockDim.x) {
      int r = e / kT, c = e % kT;
      int64_t t = t0 + r;
      float va = 0.f, vb = 0.f;
      if (t < t_end) {
        if (i0 + c < d) va = to_f32(X[t * d + i0 + c]);
        if (j0 + c < d) vb = to_f32(X[t * d + j0 + c]);
      }
      xa[r][c] = va;
      xb[r][c] = vb;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kKT; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = xa[k][ty * 4 + q];
        b[q] = xb[k][tx * 4 + q];
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
    }
    __syncthreads();
    in_chunk += kKT;
    if (in_chunk >= kChunk) {
      in_chunk = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc64[p][q] += (double)acc[p][q];
          acc[p][q] = 0.f;
        }
    }
  }
  double* out = partial + ((size_t)blockIdx.y * gridDim.x + blockIdx.x) * (kT * kT);
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) out[(ty * 4 + p) * kT + tx * 4 + q] = acc64[p][q] + (double)acc[p][q];
}

__global__ void hessian_reduce_kernel(const double* __restrict__ partial, int d, int D, int tiles,
                                      int splits, float scale, int accumulate, float* __restrict__ H) {
  int bi, bj;
  upper_tile(blockIdx.x, D, bi, bj);
  for (int e = threadIdx.x; e < kT * kT; e += blockDim.x) {
    int r = e / kT, c = e % kT;
    int i = bi * kT + r, j = bj * kT + c;
    if (i >= d || j >= d) continue;
    double s = 0.0;
    for (int k = 0; k < splits; ++k) s += partial[((size_t)k * tiles + blockIdx.x) * (kT * kT) + e];
    float v = (float)(s * (double)scale);
    float* h = H + (size_t)i * d + j;
    *h = accumulate ? *h + v : v;
  }
}

}  // namespace

size_t hessian_simt_workspace(int64_t n_tokens, int64_t d) {
  SimtPlan p = plan(n_tokens, d);
  return (size_t)p.splits * p.tiles * kT * kT * sizeof(double);
}

gptq_status hessian_simt_launch(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d, float* H,
                                float scale, int32_t accumulate, void* workspace, cudaStream_t stream) {
  SimtPlan p = plan(n_tokens, d);
  double* partial = static_cast<double*>(workspace);
  dim3 grid(p.tiles, p.splits);
  switch (x_dtype) {
    case GPTQ_FP32:
      hessian_partial_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(X), n_tokens,
                                                              (int)d, p.D, p.tokens_per_split, partial);
      break;
    case GPTQ_FP16:
      hessian_partial_kernel<__half><<<grid, 256, 0, stream>>>(static_cast<const __half*>(X), n_tokens,
                                                               (int)d, p.D, p.tokens_per_split, partial);
      break;
    case GPTQ_BF16:
      hessian_partial_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(X), n_tokens, (int)d, p.D, p.tokens_per_split, partial);
      break;
    default:
      return GPTQ_ERR_ARG;
  }
  GPTQ_LAUNCH_CHECK();
  hessian_reduce_kernel<<<p.tiles, 256, 0, stream>>>(partial, (int)d, p.D, p.tiles, p.splits, scale,
                                                     accumulate, H);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
