// Act-order ("desc_act"; zhiliyouxian blog, 实践指南; agent.csdn.net "GPTQ量化参数搜索工具", 关键参数说明):
// the columns are quantized in descending order of diag(H) (the channels with the largest calibration
// activations first), ties in column order.  The pages name the option without defining the order
// beyond "sort by activation"; descending diag(H) is the reading taken here.  The method itself does
// not change: it runs on the permuted problem H -> P H P^T, W -> W P^T, and the codes go back to the
// original column order.  Groups are consecutive steps of the quantization order.
//
//   act_order_keys_kernel     order keys of diag(H) (total order of floats as unsigned ints)
//   act_order_rank_kernel     perm[rank(i)] = i, rank = number of columns ahead of i; every CTA
//                             streams all keys through shared memory (d^2 comparisons, exact)
//   act_order_permute_kernel  H_perm[i][j] = H[min(p_i, p_j)][max(p_i, p_j)] for j >= i
//   inverse_perm_kernel       inv[perm[i]] = i, checking that perm is a permutation
//   gather_columns_kernel     W P^T in fp32 (the row staged in shared memory, gathered by perm)
//   scatter_codes_kernel      codes[:, j] = codes_in_order[:, inv[j]], four codes per thread
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kRankThreads = 256;
constexpr int kRowThreads = 256;
constexpr int kMaxRowSmem = 192 * 1024;  // largest row staged in shared memory (bytes)

// Larger float -> larger key; -0 and +0 get one key.  NaN diagonals sort as the largest (+NaN) or the
// smallest (-NaN) values; their place is otherwise unspecified.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void __launch_bounds__(256) act_order_keys_kernel(const float* __restrict__ H, int d,
                                                             uint32_t* __restrict__ keys) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < d; i += gridDim.x * blockDim.x)
    keys[i] = order_key(H[(size_t)i * d + i]);
}

// Column j comes before column i when key_j > key_i, or key_j == key_i and j < i; the rank of i is
// the number of columns before it.  Ranks of a strict total order are distinct and cover 0..d-1, so
// perm is a permutation by construction.
__global__ void __launch_bounds__(kRankThreads) act_order_rank_kernel(const uint32_t* __restrict__ keys, int d,
                                                                      int32_t* __restrict__ perm) {
  __shared__ uint32_t ks[kRankThreads];
  const int i = blockIdx.x * kRankThreads + threadIdx.x;
  const uint32_t ki = i < d ? keys[i] : 0u;
  int ahead = 0;
  for (int j0 = 0; j0 < d; j0 += kRankThreads) {
    __syncthreads();
    ks[threadIdx.x] = (j0 + threadIdx.x < d) ? keys[j0 + threadIdx.x] : 0u;
    __syncthreads();
    const int n = min(kRankThreads, d - j0);
    if (n == kRankThreads) {
#pragma unroll 16
      for (int t = 0; t < kRankThreads; ++t) {
        const uint32_t kj = ks[t];
        ahead += (kj > ki) | ((kj == ki) & (j0 + t < i));
      }
    } else {
      for (int t = 0; t < n; ++t) {
        const uint32_t kj = ks[t];
        ahead += (kj > ki) | ((kj == ki) & (j0 + t < i));
      }
    }
  }
  if (i < d) perm[ahead] = i;
}

// Upper triangle of P H P^T from the upper triangle of H.  grid.x: 256-column tiles, grid.y: rows
// (strided); tiles wholly left of the diagonal are skipped.
__global__ void __launch_bounds__(256) act_order_permute_kernel(const float* __restrict__ H, int d,
                                                                const int32_t* __restrict__ perm,
                                                                float* __restrict__ Hp) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  for (int i = blockIdx.y; i < d; i += gridDim.y) {
    if ((int)(blockIdx.x * blockDim.x + blockDim.x - 1) < i) continue;
    if (j < d && j >= i) {
      const int pi = perm[i], pj = perm[j];
      const int a = min(pi, pj), b = max(pi, pj);
      Hp[(size_t)i * d + j] = H[(size_t)a * d + b];
    }
  }
}

// inv[perm[i]] = i.  inv starts as all -1; an entry out of range or a repeated one is reported as
// GPTQ_ERR_ARG with the step i, and leaves a -1 (or the first writer) behind, which the gather and the
// scatter turn into zeros instead of reading out of bounds.
__global__ void __launch_bounds__(256) inverse_perm_kernel(const int32_t* __restrict__ perm, int d,
                                                           int32_t* __restrict__ inv, int32_t* status) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < d; i += gridDim.x * blockDim.x) {
    const int p = perm[i];
    if ((unsigned)p >= (unsigned)d) {
      report_status(status, GPTQ_ERR_ARG, i);
      continue;
    }
    if (atomicCAS(&inv[p], -1, i) != -1) report_status(status, GPTQ_ERR_ARG, i);
  }
}

// out[r][i] = float(W[r][perm[i]]); each CTA takes whole rows, staged in shared memory when they fit.
template <typename T, bool kStage>
__global__ void __launch_bounds__(kRowThreads) gather_columns_kernel(const T* __restrict__ W, int64_t m, int d,
                                                                     const int32_t* __restrict__ perm,
                                                                     float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* row_s = reinterpret_cast<T*>(smem_raw);
  for (int64_t r = blockIdx.x; r < m; r += gridDim.x) {
    const T* src = W + r * d;
    if constexpr (kStage) {
      __syncthreads();
      for (int c = threadIdx.x; c < d; c += kRowThreads) row_s[c] = src[c];
      __syncthreads();
    }
    float* dst = out + r * d;
    for (int i = threadIdx.x; i < d; i += kRowThreads) {
      const int p = perm[i];
      float v = 0.0f;
      if ((unsigned)p < (unsigned)d) v = to_f32(kStage ? row_s[p] : src[p]);
      dst[i] = v;
    }
  }
}

// codes[r][j] = in_order[r][inv[j]], four consecutive j per thread (d % 32 == 0).
template <bool kStage>
__global__ void __launch_bounds__(kRowThreads) scatter_codes_kernel(const uint8_t* __restrict__ in_order, int64_t m,
                                                                    int d, const int32_t* __restrict__ inv,
                                                                    uint8_t* __restrict__ codes) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  for (int64_t r = blockIdx.x; r < m; r += gridDim.x) {
    const uint8_t* src = in_order + r * d;
    if constexpr (kStage) {
      __syncthreads();
      for (int c = threadIdx.x * 16; c < d; c += kRowThreads * 16)
        *reinterpret_cast<uint4*>(smem_raw + c) = *reinterpret_cast<const uint4*>(src + c);
      __syncthreads();
    }
    const uint8_t* row = kStage ? smem_raw : src;
    for (int j = threadIdx.x * 4; j < d; j += kRowThreads * 4) {
      const int4 q = *reinterpret_cast<const int4*>(inv + j);
      const int qs[4] = {q.x, q.y, q.z, q.w};
      uint32_t word = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t c = ((unsigned)qs[t] < (unsigned)d) ? row[qs[t]] : 0u;
        word |= c << (8 * t);
      }
      *reinterpret_cast<uint32_t*>(codes + r * d + j) = word;
    }
  }
}

int row_grid(int64_t m) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return (int)std::min<int64_t>(m, (int64_t)sms * 8);
}

template <typename T>
gptq_status launch_gather(const void* W, int64_t m, int d, const int32_t* perm, float* out, cudaStream_t s) {
  const size_t bytes = (size_t)d * sizeof(T);
  const int grid = row_grid(m);
  if (bytes <= (size_t)kMaxRowSmem) {
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(gather_columns_kernel<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes));
    gather_columns_kernel<T, true><<<grid, kRowThreads, bytes, s>>>(static_cast<const T*>(W), m, d, perm, out);
  } else {
    gather_columns_kernel<T, false><<<grid, kRowThreads, 0, s>>>(static_cast<const T*>(W), m, d, perm, out);
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace

gptq_status act_order_launch(const float* H, int64_t d64, int32_t* perm, float* H_perm, int32_t* status,
                             cudaStream_t s) {
  const int d = (int)d64;
  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), s));
  // the keys live in the first d entries of H_perm until the permuted matrix overwrites them
  uint32_t* keys = reinterpret_cast<uint32_t*>(H_perm);
  act_order_keys_kernel<<<(d + 255) / 256, 256, 0, s>>>(H, d, keys);
  GPTQ_LAUNCH_CHECK();
  act_order_rank_kernel<<<(d + kRankThreads - 1) / kRankThreads, kRankThreads, 0, s>>>(keys, d, perm);
  GPTQ_LAUNCH_CHECK();
  dim3 grid((d + 255) / 256, (unsigned)std::min(d, 65535));
  act_order_permute_kernel<<<grid, 256, 0, s>>>(H, d, perm, H_perm);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

size_t quantize_act_order_workspace(int64_t m, int64_t d, int block_size) {
  return quantize_workspace(m, d, block_size) + align_up((size_t)m * d * sizeof(float), 256) +
         align_up((size_t)m * d, 256) + align_up((size_t)d * sizeof(int32_t), 256);
}

gptq_status quantize_act_order_launch(const void* W, int32_t w_dtype, int64_t m, int64_t d64, const float* U_perm,
                                      const int32_t* perm, const gptq_quant_cfg& cfg, uint8_t* codes,
                                      float* scales, int32_t* zeros, int32_t* status, void* workspace,
                                      cudaStream_t s) {
  const int d = (int)d64;
  char* ws = static_cast<char*>(workspace);
  size_t off = quantize_workspace(m, d, cfg.block_size);
  float* w_perm = reinterpret_cast<float*>(ws + off);
  off += align_up((size_t)m * d * sizeof(float), 256);
  uint8_t* codes_in_order = reinterpret_cast<uint8_t*>(ws + off);
  off += align_up((size_t)m * d, 256);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + off);

  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), s));
  GPTQ_CUDA_TRY(cudaMemsetAsync(inv, 0xff, (size_t)d * sizeof(int32_t), s));
  inverse_perm_kernel<<<(d + 255) / 256, 256, 0, s>>>(perm, d, inv, status);
  GPTQ_LAUNCH_CHECK();
  gptq_status st;
  switch (w_dtype) {
    case GPTQ_FP32: st = launch_gather<float>(W, m, d, perm, w_perm, s); break;
    case GPTQ_FP16: st = launch_gather<__half>(W, m, d, perm, w_perm, s); break;
    case GPTQ_BF16: st = launch_gather<__nv_bfloat16>(W, m, d, perm, w_perm, s); break;
    default: return GPTQ_ERR_ARG;
  }
  if (st != GPTQ_OK) return st;
  gptq_quant_cfg plain = cfg;
  plain.flags &= ~GPTQ_FLAG_ACT_ORDER;
  st = quantize_launch(w_perm, GPTQ_FP32, m, d, U_perm, plain, codes_in_order, scales, zeros, status, workspace, s,
                       /*clear_status=*/false);
  if (st != GPTQ_OK) return st;
  const int grid = row_grid(m);
  if (d <= kMaxRowSmem) {
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(scatter_codes_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, d));
    scatter_codes_kernel<true><<<grid, kRowThreads, d, s>>>(codes_in_order, m, d, inv, codes);
  } else {
    scatter_codes_kernel<false><<<grid, kRowThreads, 0, s>>>(codes_in_order, m, d, inv, codes);
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
