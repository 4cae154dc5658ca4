// Inference with the packed weights: Y = X_in @ What^T, What[r, j] = scale[r, g] (q[r, j] - zero[r, g]),
// the codes read straight from the packed words (FDE Interviews breakdown of GPTQ, section 01, last
// paragraph: kernels that read the 3-bit weights and dequantize them on the fly).
//
// HBM-bound for a handful of input rows: every packed word is read once.  A CTA takes 32 rows x 4096
// columns (split-K over column tiles; a second kernel sums the tiles in order, so the result does not
// depend on scheduling).  Warp w owns 4 rows; lane l takes 32-column units l, l + 32, ... of the tile.
// A unit of 32 codes is exactly `bits` words of a row's bit stream (code j in bits [b j, b j + b)),
// so it is decoded from registers: one funnel shift puts code j at mantissa bits [23 - b, 23) and one
// LOP3 masks it and ORs in the exponent of 1.0, giving f_j = 1 + q_j / 2^b exactly.  Then
//   sum_j q_j x_j = 2^b (sum_j f_j x_j - sum_j x_j),
// and the unit adds scale * (sum_j q_j x_j - zero * sum_j x_j) to its row (a unit never straddles a
// group: group sizes are multiples of 32).  Three instructions per code and input row-independent
// decode work; the input values come through L1 (every warp of the CTA reads the same tile of X).
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kRowsPerWarp = 4;
constexpr int kWarps = 8;
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;
constexpr int kUnitsPerTile = 128;  // 4096 columns

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float (&v)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
    v[2 * k] = f.x, v[2 * k + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
    v[2 * k] = f.x, v[2 * k + 1] = f.y;
  }
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// 1 + q_j / 2^BITS for code j (0..31) of a unit held in w[0..BITS-1].
template <int BITS>
__device__ __forceinline__ float decode(const uint32_t (&w)[BITS], const int j) {
  constexpr int P = 23 - BITS;  // mantissa position of the code
  const int bit = BITS * j, k = bit >> 5, s = bit & 31;
  uint32_t v;
  if (s >= P) {
    const uint32_t hi = (k + 1 < BITS) ? w[k + 1] : 0u;
    v = __funnelshift_r(w[k], hi, s - P);
  } else {
    const uint32_t lo = (k > 0) ? w[k - 1] : 0u;
    v = __funnelshift_l(lo, w[k], P - s);
  }
  return __uint_as_float((v & (((1u << BITS) - 1u) << P)) | 0x3F800000u);
}

template <int BITS, int NB, typename TX>
__global__ void __launch_bounds__(kWarps * 32) dequant_matmul_kernel(const uint32_t* __restrict__ packed,
                                                                     const float* __restrict__ scales,
                                                                     const int32_t* __restrict__ zeros, int m,
                                                                     int d, int group_size,
                                                                     const TX* __restrict__ X, int64_t ldx,
                                                                     float* __restrict__ partial, int batch) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
  const int n_units = d >> 5;
  const int u_begin = blockIdx.y * kUnitsPerTile;
  const int u_end = min(n_units, u_begin + kUnitsPerTile);
  const int wpr = (d >> 5) * BITS;  // words per row
  const int ng = group_size ? d / group_size : 1;
  const int upg = group_size ? group_size >> 5 : n_units;
  float acc[kRowsPerWarp][NB];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.0f;

  for (int u = u_begin + lane; u < u_end; u += 32) {
    uint32_t w[kRowsPerWarp][BITS];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int row = row0 + r;
#pragma unroll
      for (int k = 0; k < BITS; ++k)
        w[r][k] = (row < m) ? __ldg(packed + (int64_t)row * wpr + (int64_t)u * BITS + k) : 0u;
    }
    float part[kRowsPerWarp][NB], xs[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      xs[b] = 0.0f;
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) part[r][b] = 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float xv[NB][8];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        load8<TX>(X + b * ldx + (int64_t)u * 32 + 8 * q, xv[b]);
#pragma unroll
        for (int t = 0; t < 8; ++t) xs[b] += xv[b][t];
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const float f = decode<BITS>(w[r], 8 * q + t);
#pragma unroll
          for (int b = 0; b < NB; ++b) part[r][b] = fmaf(f, xv[b][t], part[r][b]);
        }
      }
    }
    const int g = u / upg;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int row = row0 + r;
      if (row < m) {
        const float sc = __ldg(scales + (int64_t)row * ng + g);
        const float z = (float)__ldg(zeros + (int64_t)row * ng + g);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float qx = (part[r][b] - xs[b]) * (float)(1 << BITS);  // sum_j q_j x_j
          acc[r][b] = fmaf(sc, fmaf(-z, xs[b], qx), acc[r][b]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float v = acc[r][b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[r][b] = v;
    }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int row = row0 + r;
      if (row < m) {
#pragma unroll
        for (int b = 0; b < NB; ++b) partial[((int64_t)blockIdx.y * batch + b) * m + row] = acc[r][b];
      }
    }
  }
}

// Y[b][r] = sum over column tiles of the partial sums, in tile order.
__global__ void __launch_bounds__(256) dequant_reduce_kernel(const float* __restrict__ partial, int tiles,
                                                             int64_t n, float* __restrict__ Y, int64_t ldy, int m,
                                                             int b0) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int t = 0; t < tiles; ++t) s += partial[t * n + e];
    const int64_t b = e / m, r = e % m;
    Y[(b0 + b) * ldy + r] = s;
  }
}

template <int BITS, typename TX>
void launch_chunk(int nb, dim3 grid, const uint32_t* packed, const float* scales, const int32_t* zeros, int m, int d,
                  int gs, const TX* X, int64_t ldx, float* partial, cudaStream_t s) {
  switch (nb) {
    case 1: dequant_matmul_kernel<BITS, 1, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 1); break;
    case 2: dequant_matmul_kernel<BITS, 2, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 2); break;
    case 3: dequant_matmul_kernel<BITS, 3, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 3); break;
    default: dequant_matmul_kernel<BITS, 4, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 4); break;
  }
}

template <typename TX>
gptq_status launch_typed(const int32_t* packed, const float* scales, const int32_t* zeros, int m, int d, int bits,
                         int gs, const void* Xv, int64_t batch, float* Y, float* partial, cudaStream_t s) {
  const TX* X = static_cast<const TX*>(Xv);
  const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);
  const int tiles = (d / 32 + kUnitsPerTile - 1) / kUnitsPerTile;
  dim3 grid((m + kRowsPerCta - 1) / kRowsPerCta, tiles);
  for (int64_t b0 = 0; b0 < batch; b0 += 4) {
    const int nb = (int)std::min<int64_t>(4, batch - b0);
    switch (bits) {
      case 2: launch_chunk<2, TX>(nb, grid, pw, scales, zeros, m, d, gs, X + b0 * d, d, partial, s); break;
      case 3: launch_chunk<3, TX>(nb, grid, pw, scales, zeros, m, d, gs, X + b0 * d, d, partial, s); break;
      case 4: launch_chunk<4, TX>(nb, grid, pw, scales, zeros, m, d, gs, X + b0 * d, d, partial, s); break;
      default: return GPTQ_ERR_ARG;
    }
    GPTQ_LAUNCH_CHECK();
    const int64_t n = (int64_t)nb * m;
    const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 8);
    dequant_reduce_kernel<<<blocks, 256, 0, s>>>(partial, tiles, n, Y, m, m, (int)b0);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

// What[r][j] = scale[r][g(j)] * (q[r][j] - zero[r][g(j)]) from the packed words, 32 codes per thread
template <typename TO, int BITS>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t* __restrict__ packed,
                                                         const float* __restrict__ scales,
                                                         const int32_t* __restrict__ zeros, int64_t m, int d,
                                                         int group_size, TO* __restrict__ out) {
  const int units = d >> 5, ng = group_size ? d / group_size : 1, upg = group_size ? group_size >> 5 : units;
  const int wpr = units * BITS;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < m * units; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / units;
    const int u = (int)(e % units);
    uint32_t w[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = packed[r * wpr + (int64_t)u * BITS + k];
    const float sc = scales[r * ng + u / upg], z = (float)zeros[r * ng + u / upg];
    TO* dst = out + r * d + (int64_t)u * 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float q = (decode<BITS>(w, j) - 1.0f) * (float)(1 << BITS);  // exact: q = 2^b (f - 1)
      dst[j] = from_f32<TO>(sc * (q - z));
    }
  }
}

}  // namespace

size_t dequant_matmul_workspace(int64_t m, int64_t d, int64_t batch) {
  const int64_t tiles = (d / 32 + kUnitsPerTile - 1) / kUnitsPerTile;
  return align_up((size_t)tiles * (size_t)std::min<int64_t>(batch, 4) * m * sizeof(float), 256);
}

template <typename TO>
gptq_status dequantize_typed(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m, int64_t d,
                             int32_t bits, int32_t group_size, void* out, cudaStream_t s) {
  const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);
  const int64_t n = m * (d / 32);
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  TO* o = static_cast<TO*>(out);
  switch (bits) {
    case 2: dequantize_kernel<TO, 2><<<blocks, 256, 0, s>>>(pw, scales, zeros, m, (int)d, group_size, o); break;
    case 3: dequantize_kernel<TO, 3><<<blocks, 256, 0, s>>>(pw, scales, zeros, m, (int)d, group_size, o); break;
    case 4: dequantize_kernel<TO, 4><<<blocks, 256, 0, s>>>(pw, scales, zeros, m, (int)d, group_size, o); break;
    default: return GPTQ_ERR_ARG;
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

gptq_status dequantize_launch(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m, int64_t d,
                              int32_t bits, int32_t group_size, void* out, int32_t out_dtype, cudaStream_t s) {
  switch (out_dtype) {
    case GPTQ_FP16: return dequantize_typed<__half>(packed, scales, zeros, m, d, bits, group_size, out, s);
    case GPTQ_BF16: return dequantize_typed<__nv_bfloat16>(packed, scales, zeros, m, d, bits, group_size, out, s);
    case GPTQ_FP32: return dequantize_typed<float>(packed, scales, zeros, m, d, bits, group_size, out, s);
    default: return GPTQ_ERR_ARG;
  }
}

gptq_status dequant_matmul_launch(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m,
                                  int64_t d, int32_t bits, int32_t group_size, const void* X, int32_t x_dtype,
                                  int64_t batch, float* Y, void* workspace, cudaStream_t s) {
  float* partial = static_cast<float*>(workspace);
  switch (x_dtype) {
    case GPTQ_FP16:
      return launch_typed<__half>(packed, scales, zeros, (int)m, (int)d, bits, group_size, X, batch, Y, partial, s);
    case GPTQ_BF16:
      return launch_typed<__nv_bfloat16>(packed, scales, zeros, (int)m, (int)d, bits, group_size, X, batch, Y,
                                         partial, s);
    case GPTQ_FP32:
      return launch_typed<float>(packed, scales, zeros, (int)m, (int)d, bits, group_size, X, batch, Y, partial, s);
    default: return GPTQ_ERR_ARG;
  }
}

}  // namespace gptq
